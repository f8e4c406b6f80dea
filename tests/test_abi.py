"""The C-ABI library loads, exports every entry point include/kvq.h declares,
and rejects bad arguments on the host before touching a GPU.  CPU only."""
import ctypes as C
import os
import re

import pytest

import rotated_int2_kv_head_b200 as kvq
from rotated_int2_kv_head_b200 import build as kbuild
from rotated_int2_kv_head_b200.kvq import CacheDesc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvq.h")


@pytest.fixture(scope="module")
def L():
    kbuild.build()
    return kvq.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_api():
    names = declared_functions()
    for n in ["kvq_rotate_quantize_append", "kvq_decode_attention", "kvq_decode_workspace_size",
              "kvq_get_status", "kvq_debug_rotate_f32", "kvq_debug_quantize_f32"]:
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for n in declared_functions():
        assert hasattr(L, n), n


def test_only_api_symbols_are_exported():
    out = os.popen("nm -D --defined-only %s" % kbuild.LIB).read()
    ours = sorted({l.split()[-1] for l in out.splitlines() if " T " in l and "kvq" in l})
    assert ours == declared_functions()


def desc(**kw):
    d = dict(B=2, Hkv=2, head_dim=128, group=32, capacity=64, sink_fp16=0, blocks=4096,
             k_sink=0, v_sink=0, status=256)
    d.update(kw)
    return CacheDesc(d["B"], d["Hkv"], d["head_dim"], d["group"], d["capacity"], d["sink_fp16"],
                     d["blocks"], d["k_sink"], d["v_sink"], d["status"])


def append(L, cache, mode=0, rk=1024, rv=1024, perm=2048, K=8192, V=8192, T=3, seq=512):
    return L.kvq_rotate_quantize_append(C.c_void_p(K), C.c_void_p(V), T, mode, C.c_void_p(rk),
                                        C.c_void_p(rv), C.c_void_p(perm), C.byref(cache),
                                        C.c_void_p(seq), None)


def test_append_rejects_bad_arguments_on_host(L):
    assert append(L, desc(head_dim=64)) == 2              # UNSUPPORTED
    assert append(L, desc(group=16)) == 2
    assert append(L, desc(capacity=40)) == 1              # not a multiple of 16
    assert append(L, desc(blocks=0)) == 1
    assert append(L, desc(blocks=4100)) == 2              # misaligned
    assert append(L, desc(sink_fp16=4)) == 1              # sinks without buffers
    assert append(L, desc(sink_fp16=65, k_sink=64, v_sink=64)) == 1
    assert append(L, desc(), rk=0) == 1                   # dense needs R
    assert append(L, desc(), mode=1, perm=0) == 1         # FWHT needs perm
    assert append(L, desc(), mode=7) == 1
    assert append(L, desc(), K=0) == 1
    assert append(L, desc(), K=8200) == 2
    assert append(L, desc(), T=-1) == 1
    assert append(L, desc(), T=65) == 1                   # T > capacity
    assert append(L, desc(), T=0) == 0                    # nothing to do
    assert L.kvq_rotate_quantize_append(None, None, 1, 0, None, None, None, None, None, None) == 1


def test_decode_rejects_bad_arguments_on_host(L):
    def dec(cache, Hq=2, sink=0, max_ctx=64, ws=4096, wsb=1 << 20, Q=8192, out=8192, seq=512):
        return L.kvq_decode_attention(C.c_void_p(Q), Hq, C.byref(cache), 0, C.c_void_p(1024),
                                      C.c_void_p(1024), None, C.c_void_p(seq), sink, max_ctx,
                                      C.c_void_p(ws), wsb, C.c_void_p(out), None)
    assert dec(desc(), Hq=3) == 1          # Hq not a multiple of Hkv
    assert dec(desc(), Hq=6) == 2          # G = 3 unsupported
    assert dec(desc(), Hq=32) == 2         # G = 16 unsupported
    assert dec(desc(), sink=2) == 1        # sink count mismatch
    assert dec(desc(), max_ctx=0) == 1
    assert dec(desc(), max_ctx=65) == 1
    assert dec(desc(), ws=4100) == 2       # workspace alignment
    assert dec(desc(), Q=0) == 1


def test_workspace_size_is_monotone_and_validated(L):
    f = L.kvq_decode_workspace_size
    assert f(0, 1, 1, 10, 148) == 0
    assert f(1, 3, 2, 10, 148) == 0
    a = f(1, 32, 32, 32768, 148)
    b = f(64, 32, 32, 65536, 148)
    assert 0 < a < b
    assert f(8, 32, 8, 131072, 148) % 256 == 0


def test_cache_bytes(L):
    assert L.kvq_cache_bytes(1, 32, 32768) == 32 * 2048 * 1536
    assert L.kvq_cache_bytes(1, 1, 17) == 0


def test_step_calls_reject_bad_arguments_on_host(L):
    """kvq_append_decode and kvq_append_decode_host check every argument of
    both halves before anything reaches the GPU."""
    def dev(cache, T=1, Hq=2, K=8192, Q=8192, ws=4096, max_ctx=64, out=8192):
        return L.kvq_append_decode(K, K, T, Q, Hq, C.byref(cache), 0, 1024, 1024, None, 512,
                                   max_ctx, ws, 1 << 24, out, None)

    def host(cache, T=1, Hq=2, K=8192, Q=8192, ws=4096, out=8192):
        return L.kvq_append_decode_host(K, K, T, Q, Hq, C.byref(cache), 0, 1024, 1024, None, 512,
                                        64, ws, 1 << 24, out, None)

    assert dev(desc(head_dim=64)) == 2         # UNSUPPORTED
    assert dev(desc(), K=0) == 1               # append half: no rows
    assert dev(desc(), T=65) == 1              # T > capacity
    assert dev(desc(), Q=0) == 1               # decode half: no queries
    assert dev(desc(), ws=4100) == 2           # workspace alignment
    assert dev(desc(), Hq=3) == 1              # Hq not a multiple of Hkv
    assert dev(desc(), Hq=6) == 2              # G = 3
    assert dev(desc(), max_ctx=0) == 1
    assert dev(desc(), max_ctx=65) == 1
    assert host(desc(head_dim=64)) == 2
    assert host(desc(), K=0) == 1
    assert host(desc(), out=0) == 1
    assert host(desc(), T=0) == 1              # the host step always carries rows
    assert host(desc(), ws=4100) == 2
    assert host(desc(), Hq=3) == 1


def test_step_workspace_size(L):
    f, g = L.kvq_step_workspace_size, L.kvq_decode_workspace_size
    assert f(1, 0, 32, 32, 32768, 148) == 0
    assert f(0, 1, 32, 32, 32768, 148) == 0
    for B, T, Hq, Hkv in [(1, 1, 32, 32), (8, 3, 32, 8), (64, 128, 32, 32)]:
        n, d = f(B, T, Hq, Hkv, 32768, 148), g(B, Hq, Hkv, 32768, 148)
        assert n % 256 == 0
        # the decode workspace, then K, V [B][T][Hkv][128] and Q, out [B][Hq][128] in fp16
        assert n >= d + 2 * B * T * Hkv * 256 + 2 * B * Hq * 256


def test_prerope_and_sink_calls_reject_bad_arguments_on_host(L):
    """The pre-RoPE pair, its workspace size and sink identification check
    their arguments on the host before any launch."""
    def papp(cache, T=3, gh=1, K=8192, perm=2048):
        return L.kvq_prerope_append(K, K, T, gh, perm, C.byref(cache), 512, None)

    assert papp(desc(head_dim=64)) == 2
    assert papp(desc(), gh=3) == 2               # group of 3 heads
    assert papp(desc(), gh=4) == 2               # 4 does not divide Hkv = 2
    assert papp(desc(), perm=0) == 1
    assert papp(desc(), perm=2052) == 2          # perm off its 16-byte alignment
    assert papp(desc(), T=-1) == 1
    assert papp(desc(), T=0) == 0                # nothing to do
    assert papp(desc(), K=0) == 1
    assert papp(desc(), K=8200) == 2
    assert papp(desc(), T=65) == 1               # T > capacity

    def pdec(cache, Hq=2, gh=1, Q=8192, ws=4096, base=10000.0, max_ctx=64):
        return L.kvq_prerope_decode(Q, Hq, C.byref(cache), gh, 2048, base, 512, max_ctx, ws,
                                    1 << 24, 8192, None)

    assert pdec(desc(), gh=3) == 2
    assert pdec(desc(), Q=0) == 1
    assert pdec(desc(), ws=4100) == 2
    assert pdec(desc(), Hq=3) == 1
    assert pdec(desc(), Hq=16, gh=2) == 2        # G * group_heads = 16 > 8
    assert pdec(desc(), base=1.0) == 1           # RoPE base must exceed 1
    assert pdec(desc(), base=float("nan")) == 1
    assert pdec(desc(), max_ctx=0) == 1
    assert pdec(desc(), max_ctx=65) == 1

    f = L.kvq_prerope_workspace_size
    assert f(1, 32, 32, 3, 32768, 148) == 0      # group of 3 heads
    assert f(1, 32, 32, 1, 0, 148) == 0
    assert f(1, 32, 32, 1, 32768, 148) > 0

    def ident(cache, act=8192, T=4, tau=100.0):
        return L.kvq_identify_sinks(act, T, tau, C.byref(cache), 512, None)

    with_sinks = dict(sink_fp16=4, k_sink=8192, v_sink=8192)
    assert ident(desc(**with_sinks)) == 1        # no sink list in the descriptor
    d = desc(**with_sinks)
    d.sink_pos, d.sink_count = 1024, 1536
    assert ident(d, act=0) == 1
    assert ident(d, T=0) == 1
    assert ident(d, act=8194) == 2               # act off its 4-byte alignment
    assert ident(d, T=65) == 1                   # T > capacity
    d.sink_count = None
    assert ident(d) == 1                         # a sink list without its counts


def test_binding_checks_rotation_shapes_before_calling_the_library(L):
    """Every binding that passes rotations to the library checks their dtype
    and shape first: the C ABI receives bare pointers, so an undersized R_k,
    R_v or perm would otherwise be read out of bounds by the kernels.  Runs on
    CPU: the check fires before any tensor reaches the library."""
    import torch
    cache = kvq.KVCache(1, 2, 64, device="cpu")
    good = torch.zeros((2, 128, 128), dtype=torch.float32)
    short = torch.zeros((1, 128, 128), dtype=torch.float32)
    half = torch.zeros((2, 128, 128), dtype=torch.float16)
    perm_short = torch.zeros((2, 1, 128), dtype=torch.int32)
    Q = torch.zeros((1, 2, 128), dtype=torch.float16)
    sl = torch.zeros(1, dtype=torch.int32)
    ws = torch.zeros(64, dtype=torch.uint8)
    ev = object()
    calls = {
        "decode": lambda rk, rv, pm, mode: kvq.kvq_decode_attention(
            Q, cache, mode, rk, rv, pm, sl, 0, 64, ws, Q),
        "decode_ex": lambda rk, rv, pm, mode: kvq.kvq_decode_attention_ex(
            Q[:, :, None], cache, mode, rk, rv, pm, sl, 0, 64, ws, Q[:, :, None]),
        "decode_timed": lambda rk, rv, pm, mode: kvq.kvq_decode_attention_timed(
            Q, cache, mode, rk, rv, pm, sl, 0, 64, ws, Q, ev, ev),
        "decode_noalloc": lambda rk, rv, pm, mode: kvq.kvq_decode_attention_noalloc(
            Q, cache, mode, rk, rv, pm, sl, 0, 64, Q),
        "append": lambda rk, rv, pm, mode: kvq.kvq_rotate_quantize_append(
            Q[:, None], Q[:, None], mode, rk, rv, pm, cache, sl),
        "append_decode": lambda rk, rv, pm, mode: kvq.kvq_append_decode(
            Q[:, None], Q[:, None], Q, cache, mode, rk, rv, pm, sl, 64, ws, Q),
        "append_decode_host": lambda rk, rv, pm, mode: kvq.kvq_append_decode_host(
            Q[:, None], Q[:, None], Q, cache, mode, rk, rv, pm, sl, 64, ws, Q),
    }
    for name, call in calls.items():
        with pytest.raises(ValueError, match="R_k must have shape"):
            call(short, good, None, 0)
        with pytest.raises(ValueError, match="R_v must have shape"):
            call(good, short, None, 0)
        with pytest.raises(TypeError, match="R_k must be torch.float32"):
            call(half, good, None, 0)
        with pytest.raises(ValueError, match="needs R_k and R_v"):
            call(None, good, None, 0)
        with pytest.raises(ValueError, match="perm must have shape"):
            call(None, None, perm_short, 1)
        with pytest.raises(ValueError, match="needs perm"):
            call(None, None, None, 1)
        with pytest.raises(ValueError, match="unknown rotation mode"):
            call(good, good, None, 2)


def test_debug_wait_timeout_rejects_bad_calls(L):
    ok = C.c_void_p(4096)
    assert L.kvq_debug_wait_timeout(None, 8, ok, ok, None) == 1
    assert L.kvq_debug_wait_timeout(ok, 0, ok, ok, None) == 1
    assert L.kvq_debug_wait_timeout(ok, 8, None, ok, None) == 1
    assert L.kvq_debug_wait_timeout(C.c_void_p(4104), 8, ok, ok, None) == 2
