"""The workloads at full size, in the launch configuration bench.py
uses, checked against the CPU oracle on sampled (sequence, KV head) units.

The GPU fills the whole cache from inputs drawn on the GPU; the rows of the
sampled units are copied to the host and the oracle builds its own cache
for them from the same tensors (the oracle never reads anything the CUDA
path produced), then decodes.  Properties that hold at any size are checked
on every output (finite, zero status).
"""
import numpy as np
import pytest
import torch

import rotated_int2_kv_head_b200 as kvq
import workloads as W
from oracle import oracle as orc

from kvq_testlib import rel_err

pytestmark = pytest.mark.gpu
DEC_TOL = 2e-3
CHUNK = 2048


@pytest.fixture(scope="module", autouse=True)
def built():
    from rotated_int2_kv_head_b200 import build
    build.build()


def run_workload(w, samples, prefill_to=None):
    """Fill the GPU cache to each sequence's length (all sequences are
    appended together up to the longest; shorter ones simply decode fewer
    tokens), append the step's tokens, decode.  Returns GPU outputs and the
    oracle outputs of the sampled (b, h) units."""
    dev = "cuda"
    lens = w.seq_lens().astype(np.int64)
    L = int(lens.max())
    T = w.append_T
    cap = ((L + 15) // 16) * 16
    Rk, Rv, perm = W.rotations(w)
    rk = torch.from_numpy(Rk).to(dev) if Rk is not None else None
    rv = torch.from_numpy(Rv).to(dev) if Rv is not None else None
    pm = torch.from_numpy(perm).to(dev) if perm is not None else None
    cache = kvq.KVCache(w.B, w.Hkv, cap, w.sink)
    sl = torch.zeros(w.B, dtype=torch.int32, device=dev)
    # host copies of the sampled units' rows: {(b, h): (K rows, V rows)}
    keep = {u: ([], []) for u in samples}
    pre = L - T
    for t0 in list(range(0, pre, CHUNK)) + [pre]:
        t1 = min(pre, t0 + CHUNK) if t0 < pre else L
        if t1 <= t0:
            continue
        K, V = W.kv_batch(w, t0, t1, dev)
        kvq.kvq_rotate_quantize_append(K, V, w.mode, rk, rv, pm, cache, sl)
        for (b, h), (kl, vl) in keep.items():
            kl.append(W.f16_bits(K[b, :, h]))
            vl.append(W.f16_bits(V[b, :, h]))
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(cache) == 0
    assert (sl.cpu().numpy() == L).all()
    lens_t = torch.from_numpy(lens.astype(np.int32)).to(dev)
    Q = W.queries(w, dev)
    ws = kvq.decode_workspace(w.B, w.Hq, w.Hkv, L)
    ws.fill_(0xFF)                           # uninitialised by contract: poison it
    out = torch.empty_like(Q)
    kvq.kvq_decode_attention(Q, cache, w.mode, rk, rv, pm, lens_t, w.sink, L, ws, out)
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(cache) == 0
    assert torch.isfinite(out).all()
    out = out.float().cpu().numpy()
    Qh = W.f16_bits(Q)
    refs = {}
    for (b, h), (kl, vl) in keep.items():
        Lb = int(lens[b])
        k = np.concatenate(kl)[:Lb].reshape(1, Lb, 1, 128)
        v = np.concatenate(vl)[:Lb].reshape(1, Lb, 1, 128)
        oc = orc.Cache(1, 1, cap, w.sink)
        s1 = np.zeros(1, np.int32)
        orc.append(oc, k, v, w.mode, Rk[h:h + 1] if Rk is not None else None,
                   Rv[h:h + 1] if Rv is not None else None,
                   perm[:, h:h + 1] if perm is not None else None, s1)
        q = Qh[b:b + 1, h * w.G:(h + 1) * w.G]
        ref, st = orc.decode(oc, q, w.mode, Rk[h:h + 1] if Rk is not None else None,
                             Rv[h:h + 1] if Rv is not None else None,
                             perm[:, h:h + 1] if perm is not None else None,
                             np.array([Lb], np.int32), n_threads=8)
        assert st == 0
        refs[(b, h)] = ref[0]
    return out, refs


def check(w, samples):
    out, refs = run_workload(w, samples)
    for (b, h), ref in refs.items():
        got = out[b, h * w.G:(h + 1) * w.G]
        err = rel_err(got, ref)
        assert err.max() <= DEC_TOL, ((b, h), err.max())


def test_tiny_full():
    check(W.WORKLOADS["tiny"], [(0, 0)])


def test_llama7b_full():
    check(W.WORKLOADS["llama7b"], [(0, 0), (0, 17), (0, 31)])


def test_hadamard_full():
    check(W.WORKLOADS["hadamard"], [(0, 0), (7, 13), (15, 31)])


def test_gqa_sinks_full():
    check(W.WORKLOADS["gqa_sinks"], [(0, 0), (7, 7)])


def test_gqa8_full():
    check(W.WORKLOADS["gqa8"], [(0, 0), (3, 7)])


def test_ragged_full():
    w = W.WORKLOADS["ragged"]
    lens = w.seq_lens()
    bmin, bmax = int(np.argmin(lens)), int(np.argmax(lens))
    check(w, [(bmin, 0), (bmax, 31), (5, 7)])


def test_ragged_prefill_append_full():
    """The bulk prefill append (B=4, 32768 tokens x 32 heads): sampled
    (sequence, head, token) rows of the GPU cache equal the oracle quantizer
    applied to the GPU's own rotation of the same rows, and agree with the
    oracle's rotation except at near ties."""
    w0 = W.WORKLOADS["ragged"]
    B, T = w0.extra["prefill_B"], w0.extra["prefill_T"]
    w = W.custom(name="ragged_prefill", seed=w0.seed + 1, B=B, Hq=32, Hkv=32, mode=0,
                 k_outliers=8, context=T)
    Rk, Rv, _ = W.rotations(w)
    rk, rv = torch.from_numpy(Rk).cuda(), torch.from_numpy(Rv).cuda()
    K, V = W.kv_batch(w, 0, T, "cuda")
    cache = kvq.KVCache(B, 32, T, 0)
    sl = torch.zeros(B, dtype=torch.int32, device="cuda")
    kvq.kvq_rotate_quantize_append(K, V, 0, rk, rv, None, cache, sl)
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(cache) == 0 and (sl.cpu().numpy() == T).all()
    rng = np.random.default_rng(3)
    picks = [(b, h, t) for b, h, t in zip(rng.integers(0, B, 64), rng.integers(0, 32, 64),
                                          rng.integers(0, T, 64))] + [(0, 0, 0), (B - 1, 31, T - 1)]
    blocks = cache.block_view()
    n_diff = n_codes = 0
    for b, h, t in picks:
        for kind, X, R in ((0, K, Rk), (1, V, Rv)):
            x = X[b, t, h][None].contiguous()
            # the bulk append ran the tensor-core kernel: same rotation here
            grot = kvq.kvq_debug_rotate_f32(x, 0, R=(rk if kind == 0 else rv)[h].contiguous(),
                                            variant=1)
            c, s, z = orc.quantize_rows(grot.cpu().numpy())
            blk = blocks[b, h, t // 16].cpu().numpy()
            kb, vb, ks, kz, vs, vz = orc.load_token(blk, t % 16)
            got_c = orc.unpack_row(kb if kind == 0 else vb)
            assert np.array_equal(got_c, c[0])
            assert np.array_equal(ks if kind == 0 else vs, s[0])
            assert np.array_equal(kz if kind == 0 else vz, z[0])
    # near ties against the oracle's own (fp64) rotation: the oracle appends
    # 4096 consecutive tokens of two (sequence, head) units, 2,097,152 codes,
    # and at most 1e-4 of them may differ from the GPU's
    for b, h, t0 in ((0, 0, 0), (B - 1, 31, T - 4096)):
        oc = orc.Cache(1, 1, 4096, 0)
        osl = np.zeros(1, np.int32)
        assert orc.append(oc, W.f16_bits(K[b:b + 1, t0:t0 + 4096, h:h + 1]),
                          W.f16_bits(V[b:b + 1, t0:t0 + 4096, h:h + 1]), 0, Rk[h:h + 1],
                          Rv[h:h + 1], None, osl) == 0
        g = blocks[b, h, t0 // 16:(t0 + 4096) // 16].cpu().numpy()
        x = np.bitwise_xor(g[:, :1024], oc.blocks[0, 0, :, :1024])
        n_diff += int(sum(bin((v | (v >> 1)) & 0x55).count("1") * int(c)
                          for v, c in enumerate(np.bincount(x.reshape(-1), minlength=256))))
        n_codes += 4096 * 2 * 128
    assert n_codes >= 1_000_000
    assert n_diff <= 1e-4 * n_codes, (n_diff, n_codes)


def test_gqa_sinks_identified_full():
    """gqa_sinks with its fp16 rows given to the massive tokens (identified
    before each chunk is appended), at full size; the oracle identifies and
    appends the sampled units' tokens from the same activations and rows."""
    w = W.WORKLOADS["gqa_sinks_identified"]
    dev = "cuda"
    L = int(w.context)
    Rk, Rv, _ = W.rotations(w)
    rk, rv = torch.from_numpy(Rk).to(dev), torch.from_numpy(Rv).to(dev)
    cache = kvq.KVCache(w.B, w.Hkv, L, w.sink, identified_sinks=True)
    sl = torch.zeros(w.B, dtype=torch.int32, device=dev)
    samples = [(0, 0), (5, 7)]
    keep = {u: ([], []) for u in samples}
    for t0 in range(0, L, 8192):
        t1 = min(L, t0 + 8192)
        K, V = W.kv_batch(w, t0, t1, dev)
        act = np.stack([W.activations(w, b, t0, t1) for b in range(w.B)])
        kvq.kvq_identify_sinks(torch.from_numpy(act).to(dev), W.MASSIVE_TAU, cache, sl)
        kvq.kvq_rotate_quantize_append(K, V, 0, rk, rv, None, cache, sl)
        for (b, h), (kl, vl) in keep.items():
            kl.append(W.f16_bits(K[b, :, h]))
            vl.append(W.f16_bits(V[b, :, h]))
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(cache) == 0
    lens = torch.full((w.B,), L, dtype=torch.int32, device=dev)
    Q = W.queries(w, dev)
    ws = kvq.decode_workspace(w.B, w.Hq, w.Hkv, L)
    ws.fill_(0xFF)
    out = torch.empty_like(Q)
    kvq.kvq_decode_attention(Q, cache, 0, rk, rv, None, lens, w.sink, L, ws, out)
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(cache) == 0 and torch.isfinite(out).all()
    out = out.float().cpu().numpy()
    Qh = W.f16_bits(Q)
    counts = cache.sink_count.cpu().numpy()
    for (b, h), (kl, vl) in keep.items():
        oc = orc.Cache(1, 1, L, w.sink, identified=True)
        s1 = np.zeros(1, np.int32)
        orc.identify_sinks(oc, W.activations(w, b, 0, L)[None], W.MASSIVE_TAU, s1)
        assert oc.sink_count[0] == counts[b]
        assert np.array_equal(oc.sink_pos[0], cache.sink_pos[b].cpu().numpy())
        orc.append(oc, np.concatenate(kl).reshape(1, L, 1, 128),
                   np.concatenate(vl).reshape(1, L, 1, 128), 0, Rk[h:h + 1], Rv[h:h + 1], None, s1)
        ref, st = orc.decode(oc, Qh[b:b + 1, h * w.G:(h + 1) * w.G], 0, Rk[h:h + 1], Rv[h:h + 1],
                             None, np.array([L], np.int32), n_threads=8)
        assert st == 0
        err = rel_err(out[b, h * w.G:(h + 1) * w.G], ref[0])
        assert err.max() <= DEC_TOL, ((b, h), err.max())


@pytest.mark.parametrize("gh", [1, 4])
def test_prerope_llama7b_full(gh):
    """Pre-RoPE keys on the llama7b shape (B=1, 32 heads, context 32768),
    appended in 4096-token chunks; sampled head groups against the oracle's
    append + decode of the same rows (the oracle cache holds the group's gh
    heads)."""
    w = W.custom(name="llama7b_prerope", seed=1002, B=1, Hq=32, Hkv=32, mode=1, context=32768,
                 k_outliers=8)
    dev = "cuda"
    L, base = 32768, 10000.0
    perm = W.prerope_perm(w, gh)
    pt = torch.from_numpy(perm).to(dev)
    cache = kvq.KVCache(1, 32, L)
    sl = torch.zeros(1, dtype=torch.int32, device=dev)
    groups = [0, 32 // gh - 1]
    keep = {q: ([], []) for q in groups}
    for t0 in range(0, L, 4096):
        K, V = W.kv_batch(w, t0, t0 + 4096, dev)
        kvq.kvq_prerope_append(K, V, gh, pt, cache, sl)
        for q, (kl, vl) in keep.items():
            kl.append(W.f16_bits(K[0, :, q * gh:(q + 1) * gh]))
            vl.append(W.f16_bits(V[0, :, q * gh:(q + 1) * gh]))
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(cache) == 0
    Q = W.queries(w, dev)
    ws = kvq.prerope_workspace(1, 32, 32, gh, L)
    ws.fill_(0xFF)
    out = torch.empty_like(Q)
    kvq.kvq_prerope_decode(Q, cache, gh, pt, base, sl, L, ws, out)
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(cache) == 0 and torch.isfinite(out).all()
    out = out.float().cpu().numpy()
    Qh = W.f16_bits(Q)
    for q, (kl, vl) in keep.items():
        n = 128 * gh
        psub = np.stack([perm[0, q * n:(q + 1) * n],
                         perm[1, q * n:(q + 1) * n]]).astype(np.int32)   # Hkv=gh: n entries each
        oc = orc.Cache(1, gh, L, 0)
        s1 = np.zeros(1, np.int32)
        orc.append_prerope(oc, np.concatenate(kl).reshape(1, L, gh, 128),
                           np.concatenate(vl).reshape(1, L, gh, 128), gh, psub, s1)
        ref, st = orc.decode_prerope(oc, Qh[:, q * gh:(q + 1) * gh], gh, psub, base, s1,
                                     n_threads=8)
        assert st == 0
        err = rel_err(out[0, q * gh:(q + 1) * gh], ref[0])
        assert err.max() <= DEC_TOL, (q, err.max())
