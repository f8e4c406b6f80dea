"""Failure detection on the device without a fault: a bounded wait that runs
out reports KVQ_DEV_TIMEOUT in the status word and the kernel returns, with
no copy still in flight into its shared memory, and the CUDA context stays
usable.  The wait runs out because nothing ever arrives on the barrier it
waits for (a flag nothing sets); no trap, assert or bad address is used."""
import time

import numpy as np
import pytest
import torch

import rotated_int2_kv_head_b200 as kvq
import workloads as W
from oracle import oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from rotated_int2_kv_head_b200 import build
    build.build()
    torch.cuda.init()


def test_bounded_wait_gives_up_sets_status_and_drains_its_copies():
    g = torch.Generator().manual_seed(5)
    src_h = torch.randint(0, 256, (kvq.kvq.BLOCK_BYTES,), generator=g, dtype=torch.uint8)
    src = src_h.cuda()
    cache = kvq.KVCache(1, 1, 16)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    res = kvq.kvq_debug_wait_timeout(src, 64, cache.status)
    res = res.cpu().numpy()
    elapsed = time.perf_counter() - t0
    assert res[0] == 1                                   # the wait gave up
    assert res[1] == 0                                   # the copy in flight landed first
    assert res[2] == int(src_h.sum())                    # ... with the right bytes
    assert kvq.kvq_get_status(cache) == kvq.KVQ_DEV_TIMEOUT
    assert elapsed < 5.0                                 # 64 polls, each at most ~20 us asleep
    # the context still works: clear the status and run an append + decode
    kvq.kvq_clear_status(cache)
    w = W.custom(seed=8, B=1, Hq=1, Hkv=1, mode=0)
    Rk, Rv, _ = W.rotations(w)
    rk, rv = torch.from_numpy(Rk).cuda(), torch.from_numpy(Rv).cuda()
    K, V = W.kv_batch(w, 0, 16, "cpu")
    sl = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvq.kvq_rotate_quantize_append(K.cuda(), V.cuda(), 0, rk, rv, None, cache, sl)
    Q = W.queries(w, "cpu")
    out = torch.empty((1, 1, 128), dtype=torch.float16, device="cuda")
    ws = kvq.decode_workspace(1, 1, 1, 16)
    kvq.kvq_decode_attention(Q.cuda(), cache, 0, rk, rv, None, sl, 0, 16, ws, out)
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(cache) == 0
    oc = orc.Cache(1, 1, 16, 0)
    osl = np.zeros(1, np.int32)
    orc.append(oc, W.f16_bits(K), W.f16_bits(V), 0, Rk, Rv, None, osl)
    ref, _ = orc.decode(oc, W.f16_bits(Q), 0, Rk, Rv, None, osl)
    got = out.float().cpu().numpy().astype(np.float64)
    assert np.abs(got - ref).max() / np.linalg.norm(ref) <= 2e-3


def test_timeout_status_is_sticky_and_leaves_the_counter_alone():
    """Two give-ups in a row OR the same bit into status word 0 and leave
    word 1 (the append completion counter) untouched; the copy in flight
    lands both times (no stage lost)."""
    src = torch.zeros(kvq.kvq.BLOCK_BYTES, dtype=torch.uint8, device="cuda")
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    for _ in range(2):
        res = kvq.kvq_debug_wait_timeout(src, 8, status).cpu().numpy()
        assert list(res) == [1, 0, 0]
    assert int(status[0].item()) == kvq.KVQ_DEV_TIMEOUT and int(status[1].item()) == 0
