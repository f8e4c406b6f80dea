"""CUDA path (libkvq through its C ABI) against the CPU oracle, element by
element, on seeded inputs.  Tolerances:
  - codes, scales, zeros: bit-exact when both sides quantize the same
    rotated fp32 rows;
  - rotation: <= 1e-3 relative;
  - packed cache vs the oracle's own rotation: <= 1e-4 of code elements
    differ, each at a near tie;
  - decode output: max-abs error <= 2e-3 * ||o_ref||_2 per (sequence, head).
"""
import json
import os

import numpy as np
import pytest
import torch

import rotated_int2_kv_head_b200 as kvq
import workloads as W
from oracle import oracle as orc

from kvq_testlib import (D, append_variant, download_cache, f16bits, gpu_append, gpu_decode,
                         logical, near_tie_ok, rel_err, rot_tensors, upload_oracle_cache)

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quantizer_worked.json")
DEC_TOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def built():
    from rotated_int2_kv_head_b200 import build
    build.build()
    torch.cuda.init()


# --- quantizer and rotation stages -------------------------------------------------------------

def edge_rows():
    rows = []
    g = json.load(open(GOLDEN))["groups"]
    for case in g:
        rows.append(np.tile(np.array(case["x"], np.float32), 4))
    rng = np.random.default_rng(1)
    r = rng.standard_normal(D).astype(np.float32)
    r[:32] = 7.0                                       # constant group
    r[32:64] = np.linspace(-1, 2, 32)                  # exact grid
    r[64:96] = 1000.0 + rng.standard_normal(32) * 1e-3  # offset >> range
    r[96:] = rng.standard_normal(32) * 1e-6            # subnormal fp16 scale
    rows.append(r)
    rows.append(np.zeros(D, np.float32))
    rows.append(-np.ones(D, np.float32) * 0.0)
    return np.stack(rows)


def test_quantizer_bit_exact():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal((8192, D)) * rng.uniform(0.01, 100, (8192, 1))).astype(np.float32)
    x = np.concatenate([x, edge_rows()])
    codes, meta = kvq.kvq_debug_quantize_f32(torch.from_numpy(x).cuda())
    codes = codes.cpu().numpy()
    meta = meta.cpu().numpy().view(np.uint16)
    oc, os_, oz = orc.quantize_rows(x)
    packed = np.stack([orc.pack_row(c) for c in oc])
    assert np.array_equal(codes, packed)
    assert np.array_equal(meta[:, :, 0], os_)
    assert np.array_equal(meta[:, :, 1], oz)


@pytest.mark.parametrize("mode,variant", [(0, 0), (0, 1), (1, 0), (1, 1)])
def test_rotation_stage(mode, variant):
    """variant 0: the small-batch append kernel's rotation; 1: the bulk
    kernel's (dense: tcgen05 with R as fp16 hi + lo), over 3000 rows =
    23 full 128-row tiles and a ragged one."""
    w = W.custom(seed=3, Hkv=1, mode=mode, k_outliers=8)
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((3000, D)) * 3).astype(np.float16)
    x[:, :8] *= 20
    rt, rn = rot_tensors(w)
    X = torch.from_numpy(x).cuda()
    if mode == 0:
        got = kvq.kvq_debug_rotate_f32(X, 0, R=rt[0][0].contiguous(), variant=variant)
        ref = orc.rotate_rows_f32(x.view(np.uint16), 0, R=rn[0][0])
    else:
        got = kvq.kvq_debug_rotate_f32(X, 1, perm=rt[2][0, 0].contiguous())
        ref = orc.rotate_rows_f32(x.view(np.uint16), 1, perm=rn[2][0, 0])
    got = got.cpu().numpy()
    err = np.abs(got - ref).max(axis=1) / np.abs(ref).max(axis=1)
    assert err.max() <= 1e-3
    assert err.max() <= 1e-5        # fp32 arithmetic: far inside the bound


# --- append ---------------------------------------------------------------------------------------

def run_append(w, L0, T, device="cuda"):
    """Append T tokens at lengths L0 on both sides; return everything."""
    rt, rn = rot_tensors(w)
    B = w.B
    K = torch.stack([W.kv_rows(w, b, L0[b], L0[b] + T, "cpu")[0] for b in range(B)])
    V = torch.stack([W.kv_rows(w, b, L0[b], L0[b] + T, "cpu")[1] for b in range(B)])
    cap = ((max(L0) + T + 15) // 16) * 16 + 16
    cache = kvq.KVCache(B, w.Hkv, cap, w.sink)
    sl = torch.tensor(L0, dtype=torch.int32, device=device)
    gpu_append(cache, K.cuda(), V.cuda(), w, rt, sl)
    oc = orc.Cache(B, w.Hkv, cap, w.sink)
    osl = np.array(L0, np.int32)
    st = orc.append(oc, f16bits(K), f16bits(V), w.mode, rn[0], rn[1], rn[2], osl)
    assert st == 0
    assert list(sl.cpu().numpy()) == list(osl)
    assert kvq.kvq_get_status(cache) == 0
    return cache, oc, K, V, rt, rn


@pytest.mark.parametrize("mode,S,T,L0", [
    # CUDA-core appends (dense: T < 32 and B*T < 256 or T < 8; permutation
    # + FWHT: T < 128 and B*T < 1024 or T < 32)
    (0, 0, 1, [0, 5, 16]),
    (0, 4, 16, [0, 3, 29]),
    (0, 20, 31, [0, 2, 31]),
    (0, 4, 7, list(range(0, 80, 2))),            # B*T = 280 rows, T < 8
    (0, 0, 8, list(range(0, 62, 2))),            # B = 31: 248 rows
    (1, 0, 37, [0, 5, 16]),
    (1, 4, 1, [3, 0, 21]),
    (1, 0, 31, list(range(0, 80, 2))),           # B*T = 1240 rows, T < 32
    # tensor-core appends of a partial tile per job: dense from T = 32, and
    # from T = 8 with B*T = 256 rows; FWHT from T = 32 with B*T = 1024
    (0, 0, 32, [0, 5, 16]),
    (0, 4, 37, [0, 3, 29]),
    (0, 20, 70, [0, 2, 31]),
    (0, 4, 8, list(range(0, 64, 2))),            # B = 32: 256 rows
    (1, 4, 32, list(range(0, 64, 2))),           # B = 32: 1024 rows
    (1, 0, 64, list(range(1, 33, 2))),           # B = 16: 1024 rows
    # bulk dense appends: T=2400 gives 228 tiles, so CTAs cross (sequence,
    # head, K|V) boundaries mid-range
    (0, 20, 520, [0, 2, 31]),
    (0, 0, 2400, [0, 7, 16]),
    # bulk permutation + FWHT appends (T >= 128): the same tensor-core kernel
    # with B built from the permutation; one full tile, and ragged tiles
    # across rotation changes
    (1, 0, 128, [0, 5, 16]),
    (1, 20, 300, [0, 2, 31]),
    (1, 0, 2400, [0, 7, 16]),
])
def test_append_matches_oracle(mode, S, T, L0):
    w = W.custom(seed=10 + T, B=len(L0), Hkv=2, mode=mode, sink=S, k_outliers=4,
                 channel_scale=(0.5, 20.0) if mode == 1 else None)
    cache, oc, K, V, rt, rn = run_append(w, L0, T)
    gc = download_cache(cache)
    # (a) exact: the GPU bytes equal the oracle quantizer applied to the GPU's
    #     own rotated rows, stored in the oracle's layout
    exp = orc.Cache(w.B, w.Hkv, oc.capacity, S)
    n_codes = n_diff = 0
    for kind, X in ((0, K), (1, V)):
        for h in range(w.Hkv):
            rows = X[:, :, h].reshape(-1, D).cuda()
            if mode == 0:
                R = (rt[0] if kind == 0 else rt[1])[h].contiguous()
                variant = append_variant(0, T, w.B)   # the kernel the append used
                grot = kvq.kvq_debug_rotate_f32(rows, 0, R=R, variant=variant).cpu().numpy()
                orot = orc.rotate_f64(orc.f16_bits_to_f32(f16bits(rows)).astype(np.float64), 0,
                                      R=(rn[0] if kind == 0 else rn[1])[h])
            else:
                pm = rt[2][kind, h].contiguous()
                grot = kvq.kvq_debug_rotate_f32(rows, 1, perm=pm,
                                                variant=append_variant(1, T, w.B)).cpu().numpy()
                orot = orc.rotate_f64(orc.f16_bits_to_f32(f16bits(rows)).astype(np.float64), 1,
                                      perm=rn[2][kind, h])
            grot = grot.reshape(w.B, T, D)
            orot = orot.reshape(w.B, T, D)
            for b in range(w.B):
                for t in range(T):
                    p = L0[b] + t
                    if p < S:
                        sink = (gc.k_sink if kind == 0 else gc.v_sink)[b, h, p]
                        assert np.array_equal(sink, orc.f32_to_f16_bits(grot[b, t]))
                        continue
                    c, s, z = orc.quantize_rows(grot[b, t])
                    lg = logical(gc, b, h, p)
                    assert np.array_equal(lg[kind], c[0])
                    assert np.array_equal(lg[2 + 2 * kind], s[0])
                    assert np.array_equal(lg[3 + 2 * kind], z[0])
                    # (b) against the oracle's own rotation: near ties only
                    lo = logical(oc, b, h, p)
                    n_codes += D
                    n_diff += int((lo[kind] != lg[kind]).sum())
                    if np.array_equal(lo[2 + 2 * kind], lg[2 + 2 * kind]) and \
                            np.array_equal(lo[3 + 2 * kind], lg[3 + 2 * kind]):
                        assert near_tie_ok(orot[b, t], lo[kind], lg[kind], lo[2 + 2 * kind],
                                           lo[3 + 2 * kind])
    # every differing code above is a near tie; the rate of such codes is
    # measured over more than a million codes per append kernel in
    # test_near_tie_rate_over_a_million_codes
    assert n_diff < n_codes
    # blocks of positions never written stay untouched (zero)
    for b in range(w.B):
        last = (L0[b] + T + 15) // 16
        assert not gc.blocks[b, :, last:].any()


# number of set 2-bit fields in each byte value: (x | x >> 1) & 0x55 keeps one
# bit per nonzero code
_NONZERO_CODES = np.array([bin((x | (x >> 1)) & 0x55).count("1") for x in range(256)], np.int64)


def code_mismatches(blocks_a, blocks_b):
    """Differing 2-bit codes between two arrays of cache blocks [..., 1536]
    (K codes in bytes [0, 512), V codes in [512, 1024) of every block)."""
    x = np.bitwise_xor(blocks_a[..., :1024], blocks_b[..., :1024])
    return int(_NONZERO_CODES[x].sum())


@pytest.mark.parametrize("mode,T", [(0, 20), (0, 37), (0, 300), (1, 37), (1, 200)])
def test_gpu_cache_reads_as_documented(mode, T):
    """The GPU's cache bytes read through the documented block format
    (tests/block_format.py: no oracle or kernel offset code): every appended
    position holds the codes and fp16 scale / zero that the oracle's
    quantizer gives for the GPU's own rotated row, and every other position
    of the cache is zero.  CUDA-core and tensor-core appends, both
    rotations."""
    from tests import block_format as bf
    w = W.custom(seed=60 + T + mode, B=2, Hkv=2, mode=mode, k_outliers=4,
                 channel_scale=(0.5, 20.0) if mode == 1 else None)
    L0 = [3, 16]
    cache, oc, K, V, rt, rn = run_append(w, L0, T)
    got = bf.read_blocks(cache.block_view().cpu().numpy())      # [B][Hkv][nblk][16] ...
    written = np.zeros(got["k"].shape[:4], bool)
    for kind, X in ((0, K), (1, V)):
        for h in range(w.Hkv):
            rows = X[:, :, h].reshape(-1, D).cuda()
            if mode == 0:
                R = (rt[0] if kind == 0 else rt[1])[h].contiguous()
                grot = kvq.kvq_debug_rotate_f32(rows, 0, R=R, variant=append_variant(0, T, w.B))
            else:
                grot = kvq.kvq_debug_rotate_f32(rows, 1, perm=rt[2][kind, h].contiguous(),
                                                variant=append_variant(1, T, w.B))
            grot = grot.cpu().numpy().reshape(w.B, T, D)
            for b in range(w.B):
                c, s, z = orc.quantize_rows(grot[b])
                p = np.arange(L0[b], L0[b] + T)
                blk, tau = p // 16, p % 16
                key = ("k", "ks", "kz") if kind == 0 else ("v", "vs", "vz")
                assert np.array_equal(got[key[0]][b, h, blk, tau], c)
                assert np.array_equal(got[key[1]][b, h, blk, tau], s)
                assert np.array_equal(got[key[2]][b, h, blk, tau], z)
                written[b, h, blk, tau] = True
    for name in ("k", "v", "ks", "kz", "vs", "vz"):
        assert not got[name][~written].any()


@pytest.mark.parametrize("path", ["dense_cuda_cores", "dense_tensor_cores", "fwht_step",
                                  "fwht_chunk", "fwht_tensor_cores", "prerope_gh4"])
def test_near_tie_rate_over_a_million_codes(path):
    """Codes that differ between the packed cache and the oracle's append of
    the same rows (its fp64 rotation) come only from near ties: at most 1e-4
    of the codes, counted over 2,097,152 codes (2048 tokens x 4 heads x K and
    V) for every append kernel - the CUDA-core dense append (16 tokens at a
    time), the tensor-core bulk append (dense, and permutation + FWHT), the
    CUDA-core FWHT append a few tokens at a time and in chunks, and the
    pre-RoPE group rotation."""
    Hkv, T = 4, 2048
    mode = 0 if path.startswith("dense") else 1
    chunk = {"dense_cuda_cores": 16, "dense_tensor_cores": T, "fwht_step": 8,
             "fwht_chunk": 64, "fwht_tensor_cores": T, "prerope_gh4": 256}[path]
    w = W.custom(seed=540 + len(path), B=1, Hq=Hkv, Hkv=Hkv, mode=mode, context=T,
                 k_outliers=8, channel_scale=(0.5, 20.0) if mode == 1 else None)
    rt, rn = rot_tensors(w)
    K, V = W.kv_batch(w, 0, T, "cuda")
    cache = kvq.KVCache(1, Hkv, T)
    sl = torch.zeros(1, dtype=torch.int32, device="cuda")
    oc = orc.Cache(1, Hkv, T, 0)
    osl = np.zeros(1, np.int32)
    if path == "prerope_gh4":
        perm = W.prerope_perm(w, 4)
        pt = torch.from_numpy(perm).cuda()
        for t0 in range(0, T, chunk):
            kvq.kvq_prerope_append(K[:, t0:t0 + chunk].contiguous(), V[:, t0:t0 + chunk].contiguous(),
                                   4, pt, cache, sl)
        assert orc.append_prerope(oc, f16bits(K), f16bits(V), 4, perm, osl) == 0
    else:
        for t0 in range(0, T, chunk):
            gpu_append(cache, K[:, t0:t0 + chunk], V[:, t0:t0 + chunk], w, rt, sl)
        assert orc.append(oc, f16bits(K), f16bits(V), mode, *rn, osl) == 0
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(cache) == 0 and int(sl.item()) == T
    n_codes = Hkv * T * 2 * D
    n_diff = code_mismatches(cache.block_view().cpu().numpy(), oc.blocks)
    assert n_codes >= 1_000_000
    assert n_diff <= 1e-4 * n_codes, (n_diff, n_codes)


def test_append_capacity_and_status():
    w = W.custom(seed=4, B=2, Hkv=1, mode=0)
    rt, _ = rot_tensors(w)
    cache = kvq.KVCache(2, 1, 32, 0)
    K = torch.randn((2, 8, 1, D), device="cuda").half()
    sl = torch.tensor([30, 2], dtype=torch.int32, device="cuda")
    gpu_append(cache, K, K, w, rt, sl)
    assert list(sl.cpu().numpy()) == [30, 10]
    assert kvq.kvq_get_status(cache) == kvq.KVQ_DEV_CAPACITY
    assert not cache.block_view()[0].any()
    kvq.kvq_clear_status(cache)
    assert kvq.kvq_get_status(cache) == 0


# --- decode ----------------------------------------------------------------------------------------

def build_oracle_cache(w, lens, cap):
    """The oracle appends every sequence's tokens [0, lens[b]) (one call per
    distinct chunk so sequences can differ in length)."""
    _, rn = rot_tensors(w)
    oc = orc.Cache(w.B, w.Hkv, cap, w.sink)
    for b in range(w.B):
        k, v = W.kv_rows(w, b, 0, lens[b], "cpu")
        sub = orc.Cache(1, w.Hkv, cap, w.sink)
        sl = np.zeros(1, np.int32)
        orc.append(sub, f16bits(k[None]), f16bits(v[None]), w.mode, rn[0], rn[1], rn[2], sl)
        oc.blocks[b] = sub.blocks[0]
        if w.sink:
            oc.k_sink[b] = sub.k_sink[0]
            oc.v_sink[b] = sub.v_sink[0]
    return oc


DECODE_CASES = [
    # G, mode, S, lengths
    (1, 0, 0, [1, 15, 16, 17, 300, 1000]),
    (1, 1, 0, [33, 512, 2047]),
    (2, 0, 4, [1, 4, 5, 19, 800]),
    (4, 0, 4, [4, 3, 20, 257, 1500]),
    (8, 1, 17, [16, 17, 18, 600]),
    (4, 1, 0, [2048, 1, 999]),
    # many sequences: up to 32 the split kernel sets its schedule up per
    # thread, above 32 through a scan over the CTA (both sides of the switch)
    (1, 0, 0, [1 + (37 * i) % 200 for i in range(32)]),
    (2, 1, 4, [1 + (53 * i) % 260 for i in range(33)]),
    (4, 0, 0, [16 * (1 + i % 7) + i % 3 for i in range(40)]),
]


@pytest.mark.parametrize("G,mode,S,lens", DECODE_CASES)
def test_decode_matches_oracle(G, mode, S, lens):
    Hkv = 2
    w = W.custom(seed=20 + G + S, B=len(lens), Hq=Hkv * G, Hkv=Hkv, mode=mode, sink=S,
                 k_outliers=6, sink_key_scale=50.0 if S else 1.0)
    cap = ((max(lens) + 15) // 16) * 16
    oc = build_oracle_cache(w, lens, cap)
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


@pytest.mark.parametrize("G,mode,q_len", [(1, 0, 1), (2, 1, 1), (4, 0, 1), (8, 1, 1), (1, 1, 4),
                                           (4, 0, 2)])
def test_interior_stage_shortcut_is_exact(G, mode, q_len):
    """The split kernel skips the position masks and the NaN guard on stages
    that lie wholly inside every query's context when the cache has no
    identified sinks.  The same bytes in a cache that lists identified sinks
    (none of them in use) take the general path on every stage: the two
    decodes must agree bit for bit."""
    Hkv = 2
    lens = [q_len, 15, 16, 64, 65, 255, 256, 257, 1000, 2049, 4100]   # each at least q_len
    w = W.custom(seed=70 + 10 * G + mode + q_len, B=len(lens), Hq=Hkv * G, Hkv=Hkv, mode=mode,
                 k_outliers=4)
    rt, _ = rot_tensors(w)
    cap = ((max(lens) + 15) // 16) * 16
    plain = kvq.KVCache(w.B, Hkv, cap, 0)
    sl = torch.zeros(w.B, dtype=torch.int32, device="cuda")
    K, V = W.kv_batch(w, 0, max(lens), "cpu")
    gpu_append(plain, K.cuda(), V.cuda(), w, rt, sl)
    listed = kvq.KVCache(w.B, Hkv, cap, 1, identified_sinks=True)
    listed.blocks.copy_(plain.blocks)
    assert not listed.sink_count.any()
    lens_t = torch.tensor(lens, dtype=torch.int32, device="cuda")
    Q = torch.randn((w.B, w.Hq, q_len, D), generator=torch.Generator().manual_seed(G + q_len)).half().cuda()
    outs = []
    for c in (plain, listed):
        ws = kvq.decode_workspace(w.B, w.Hq * q_len, Hkv, max(lens))
        out = torch.empty_like(Q)
        kvq.kvq_decode_attention_ex(Q, c, mode, rt[0], rt[1], rt[2], lens_t, c.sink_fp16, max(lens),
                                    ws, out)
        outs.append(out)
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(plain) == 0 and kvq.kvq_get_status(listed) == 0
    assert torch.isfinite(outs[0].float()).all()
    assert torch.equal(outs[0], outs[1])


def split_group_spans(B, Hkv, max_ctx, lens, S, sms):
    """Schedule slots of every group of the split kernel, from the library's
    stream-K split: min(SMs, blocks / 64) CTAs over the slots of all units
    (a non-empty unit: 8 leading slots, then one per 16-token block), each
    CTA's share cut into four contiguous group ranges."""
    blocks = B * Hkv * (-(-max_ctx // 16))
    C = max(1, min(sms, -(-blocks // 64)))
    def slots(L):
        nb = (L - 1) // 16 - S // 16 + 1 if S < L else 0
        return nb + 8 if nb > 0 else 0
    N = sum(Hkv * slots(L) for L in lens)
    W_ = max(1, -(-N // C))
    spans = []
    for c in range(C):
        beg, end = c * W_, min(N, c * W_ + W_)
        if beg >= end:
            continue
        wg = -(-(end - beg) // 4)
        spans += [min(end, p + wg) - p for p in range(beg, beg + 4 * wg, wg) if p < end]
    return spans


@pytest.mark.parametrize("G", [1, 2])
def test_staged_start_matches_oracle(G):
    """Short contexts, where every group of the split kernel has a range of
    3 to 8 stages and so takes the staged ring start (its first stage alone,
    the rest of its ring once that stage has landed), with units starting
    inside most ranges: the decode against the oracle on the same cache
    bytes, and through a paged copy of the cache (a random block table),
    whose producer is a whole warp, bit for bit the same."""
    B, Hkv = 8, 8
    lens = [int(x) for x in np.random.default_rng(500 + G).integers(3000, 14000, B)]
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    spans = split_group_spans(B, Hkv, max(lens), lens, 0, sms)
    assert sum(32 < s <= 128 for s in spans) >= 0.9 * len(spans)       # 16 blocks per stage
    w = W.custom(seed=510 + G, B=B, Hq=Hkv * G, Hkv=Hkv, mode=0, k_outliers=4)
    rt, rn = rot_tensors(w)
    cap = ((max(lens) + 15) // 16) * 16
    cache = kvq.KVCache(B, Hkv, cap, 0)
    sl = torch.zeros(B, dtype=torch.int32, device="cuda")
    for t0 in range(0, max(lens), 4096):
        K, V = W.kv_batch(w, t0, min(max(lens), t0 + 4096), "cuda")
        gpu_append(cache, K, V, w, rt, sl)
    lens_t = torch.tensor(lens, dtype=torch.int32, device="cuda")
    Q = W.queries(w, "cuda")
    out = gpu_decode(cache, Q, w, rt, lens_t, max(lens))
    nblk = cap // 16
    num_blocks = B * nblk + 5
    table = torch.randperm(num_blocks, generator=torch.Generator().manual_seed(7))[:B * nblk]
    table = table.view(B, nblk).to(torch.int32).cuda()
    paged = kvq.PagedKVCache(B, Hkv, cap, num_blocks, table, 0)
    paged.block_view()[table.view(-1).long()] = cache.block_view().permute(0, 2, 1, 3).reshape(
        B * nblk, Hkv, -1)
    assert torch.equal(paged.logical_view(), cache.block_view())
    out_p = gpu_decode(paged, Q, w, rt, lens_t, max(lens))
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(cache) == 0 and kvq.kvq_get_status(paged) == 0
    assert torch.equal(out, out_p)
    oc = download_cache(cache)
    ref, _ = orc.decode(oc, f16bits(Q.cpu()), 0, rn[0], rn[1], None, np.array(lens, np.int32))
    assert rel_err(out.float().cpu().numpy(), ref).max() <= DEC_TOL


@pytest.mark.parametrize("G,mode,S,lens", DECODE_CASES[:3])
def test_append_then_decode_end_to_end(G, mode, S, lens):
    """GPU append + GPU decode against oracle append + oracle decode."""
    Hkv = 2
    w = W.custom(seed=40 + G, B=len(lens), Hq=Hkv * G, Hkv=Hkv, mode=mode, sink=S, k_outliers=6)
    cap = ((max(lens) + 15) // 16) * 16
    oc = build_oracle_cache(w, lens, cap)
    rt, rn = rot_tensors(w)
    cache = kvq.KVCache(w.B, Hkv, cap, S)
    for b in range(w.B):     # one sequence at a time: lengths differ
        k, v = W.kv_rows(w, b, 0, lens[b], "cpu")
        k, v = k.cuda(), v.cuda()
        sub = kvq.KVCache(1, Hkv, cap, S)
        sl1 = torch.zeros(1, dtype=torch.int32, device="cuda")
        gpu_append(sub, k[None], v[None], w, rt, sl1)
        cache.block_view()[b].copy_(sub.block_view()[0])
        if S:
            cache.k_sink[b].copy_(sub.k_sink[0])
            cache.v_sink[b].copy_(sub.v_sink[0])
    Q = W.queries(w, "cpu")
    sl = np.array(lens, np.int32)
    ref, _ = orc.decode(oc, f16bits(Q), mode, rn[0], rn[1], rn[2], sl, n_threads=8)
    out = gpu_decode(cache, Q.cuda(), w, rt, torch.from_numpy(sl).cuda(), max(lens))
    err = rel_err(out.cpu().numpy(), ref)
    assert err.max() <= DEC_TOL, err.max()


def test_decode_bad_lengths_give_zero_rows_and_status():
    w = W.custom(seed=7, B=3, Hq=2, Hkv=2, mode=0)
    lens = [40, 40, 40]
    oc = build_oracle_cache(w, lens, 48)
    rt, rn = rot_tensors(w)
    cache = upload_oracle_cache(oc)
    Q = W.queries(w, "cpu")
    sl = np.array([40, 0, 49], np.int32)
    out = gpu_decode(cache, Q.cuda(), w, rt, torch.from_numpy(sl).cuda(), 48).cpu().numpy()
    assert not out[1].any() and not out[2].any()
    assert kvq.kvq_get_status(cache) == kvq.KVQ_DEV_BAD_LEN
    ref, _ = orc.decode(oc, f16bits(Q), 0, rn[0], rn[1], rn[2], sl)
    assert rel_err(out[0:1], ref[0:1]).max() <= DEC_TOL


# --- decode with several new tokens per sequence, and output in the rotated basis -----------------

MQ_CASES = [
    # G, q_len, mode, S, lengths
    (1, 2, 0, 0, [2, 17, 300, 1000]),
    (1, 4, 1, 0, [4, 33, 512]),
    (1, 8, 0, 4, [8, 9, 700]),
    (2, 2, 0, 4, [3, 40, 257]),
    (4, 2, 1, 0, [2, 1500]),
]


@pytest.mark.parametrize("G,q_len,mode,S,lens", MQ_CASES)
def test_multi_query_decode_matches_oracle(G, q_len, mode, S, lens):
    """q_len new tokens per sequence: query i sees positions [0, L - q_len + i];
    each is checked against the oracle's ordinary decode over that prefix."""
    Hkv = 2
    w = W.custom(seed=60 + 10 * G + q_len, B=len(lens), Hq=Hkv * G, Hkv=Hkv, mode=mode, sink=S,
                 k_outliers=4, sink_key_scale=50.0 if S else 1.0)
    cap = ((max(lens) + 15) // 16) * 16
    oc = build_oracle_cache(w, lens, cap)
    rt, rn = rot_tensors(w)
    g = torch.Generator().manual_seed(900 + q_len)
    Q = torch.randn((w.B, w.Hq, q_len, D), generator=g).to(torch.float16)
    cache = upload_oracle_cache(oc)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = kvq.decode_workspace(w.B, w.Hq * q_len, Hkv, max(lens))
    ws.fill_(0xFF)
    out = torch.empty_like(Q).cuda()
    kvq.kvq_decode_attention_ex(Q.cuda(), cache, mode, rt[0], rt[1], rt[2], sl, S, max(lens), ws,
                                out)
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(cache) == 0
    got = out.cpu().numpy()
    for i in range(q_len):
        li = np.array(lens, np.int32) - (q_len - 1 - i)
        ref, st = orc.decode(oc, f16bits(Q[:, :, i].contiguous()), mode, rn[0], rn[1], rn[2], li,
                             n_threads=8)
        assert st == 0
        err = rel_err(got[:, :, i], ref)
        assert err.max() <= DEC_TOL, (i, err.max())


def test_multi_query_short_sequence_gives_zero_rows_and_status():
    """A sequence shorter than q_len: the queries that would start before
    position 0 get zero rows and KVQ_DEV_BAD_LEN; the others are normal."""
    w = W.custom(seed=71, B=2, Hq=2, Hkv=2, mode=0, k_outliers=4)
    lens = [2, 50]
    q_len = 4
    cap = 64
    oc = build_oracle_cache(w, lens, cap)
    rt, rn = rot_tensors(w)
    Q = torch.randn((2, 2, q_len, D), generator=torch.Generator().manual_seed(5)).to(torch.float16)
    cache = upload_oracle_cache(oc)
    ws = kvq.decode_workspace(2, 2 * q_len, 2, 50)
    out = torch.full_like(Q, float("nan")).cuda()
    kvq.kvq_decode_attention_ex(Q.cuda(), cache, 0, rt[0], rt[1], None,
                                torch.tensor(lens, dtype=torch.int32, device="cuda"), 0, 50, ws, out)
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(cache) & kvq.KVQ_DEV_BAD_LEN
    got = out.cpu().float().numpy()
    assert (got[0, :, :2] == 0).all()                    # positions -2 and -1: no context
    for i in range(2, q_len):                            # sequence 0, queries at positions 0, 1
        ref, _ = orc.decode(oc, f16bits(Q[:, :, i].contiguous()), 0, rn[0], rn[1], None,
                            np.array([i - 1, 50 - (q_len - 1 - i)], np.int32), n_threads=4)
        assert rel_err(got[0, :, i], ref[0]).max() <= DEC_TOL
    assert np.isfinite(got[1]).all()


@pytest.mark.parametrize("mode,G,S", [(0, 1, 0), (1, 2, 4), (0, 4, 4)])
def test_decode_out_rotated(mode, G, S):
    """KVQ_DECODE_OUT_ROTATED returns o_rot: the oracle's output carried back
    into the rotated basis (out . R_v, or perm + FWHT) must match."""
    Hkv = 2
    lens = [5, 300, 1025]
    w = W.custom(seed=80 + G, B=len(lens), Hq=Hkv * G, Hkv=Hkv, mode=mode, sink=S, k_outliers=4)
    cap = ((max(lens) + 15) // 16) * 16
    oc = build_oracle_cache(w, lens, cap)
    rt, rn = rot_tensors(w)
    Q = W.queries(w, "cpu")
    sl = np.array(lens, np.int32)
    ref, st = orc.decode(oc, f16bits(Q), mode, rn[0], rn[1], rn[2], sl, n_threads=8)
    assert st == 0
    ref_rot = np.empty_like(ref)
    for b in range(w.B):
        for hq in range(w.Hq):
            h = hq // G
            if mode == 0:
                ref_rot[b, hq] = orc.rotate_f64(ref[b, hq][None], 0, R=rn[1][h])[0]
            else:
                ref_rot[b, hq] = orc.rotate_f64(ref[b, hq][None], 1, perm=rn[2][1, h])[0]
    cache = upload_oracle_cache(oc)
    ws = kvq.decode_workspace(w.B, w.Hq, Hkv, max(lens))
    out = torch.empty((w.B, w.Hq, 1, D), dtype=torch.float16, device="cuda")
    kvq.kvq_decode_attention_ex(Q.cuda()[:, :, None].contiguous(), cache, mode, rt[0], rt[1], rt[2],
                                torch.from_numpy(sl).cuda(), S, max(lens), ws, out,
                                flags=kvq.KVQ_DECODE_OUT_ROTATED)
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(cache) == 0
    err = rel_err(out[:, :, 0].cpu().numpy(), ref_rot)
    assert err.max() <= DEC_TOL, err.max()


# --- paged caches ------------------------------------------------------------------------------

@pytest.mark.parametrize("mode,S", [(0, 0), (0, 20), (1, 4)])
def test_paged_cache_matches_contiguous(mode, S):
    """The same appends into a contiguous cache and into a paged one (a random
    block table over a larger pool) give byte-identical blocks once the pool is
    gathered through the table, and bit-identical decodes.  The appends cover
    the small-batch kernel (T=37), the bulk kernel (T=300) and single tokens."""
    B, Hkv, cap = 3, 2, 1024
    nblk = cap // 16
    w = W.custom(seed=90 + mode + S, B=B, Hq=2 * Hkv, Hkv=Hkv, mode=mode, sink=S, k_outliers=4)
    rt, _ = rot_tensors(w)
    num_blocks = B * nblk + 7
    perm = torch.randperm(num_blocks, generator=torch.Generator().manual_seed(3))[:B * nblk]
    table = perm.view(B, nblk).to(torch.int32).cuda()
    flat = kvq.KVCache(B, Hkv, cap, S)
    paged = kvq.PagedKVCache(B, Hkv, cap, num_blocks, table, S)
    L0 = [0, 5, 16]
    sl_f = torch.tensor(L0, dtype=torch.int32, device="cuda")
    sl_p = sl_f.clone()
    pos = list(L0)
    for T in (37, 300, 1, 1):
        K = torch.stack([W.kv_rows(w, b, pos[b], pos[b] + T, "cpu")[0] for b in range(B)]).cuda()
        V = torch.stack([W.kv_rows(w, b, pos[b], pos[b] + T, "cpu")[1] for b in range(B)]).cuda()
        gpu_append(flat, K, V, w, rt, sl_f)
        gpu_append(paged, K, V, w, rt, sl_p)
        pos = [p + T for p in pos]
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(flat) == 0 and kvq.kvq_get_status(paged) == 0
    assert torch.equal(sl_f, sl_p)
    assert torch.equal(paged.logical_view(), flat.block_view())
    if S:
        assert torch.equal(paged.k_sink, flat.k_sink) and torch.equal(paged.v_sink, flat.v_sink)
    Q = W.queries(w, "cuda")
    out_f = gpu_decode(flat, Q, w, rt, sl_f, max(pos))
    out_p = gpu_decode(paged, Q, w, rt, sl_p, max(pos))
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(paged) == 0
    assert torch.equal(out_f, out_p)


def test_paged_bad_table_entry_sets_status():
    """A table entry outside the pool: the append skips that block and the
    decode reads pool block 0 instead; both report KVQ_DEV_BAD_TABLE."""
    B, Hkv, cap = 2, 2, 64
    w = W.custom(seed=97, B=B, Hq=Hkv, Hkv=Hkv, mode=0, k_outliers=4)
    rt, _ = rot_tensors(w)
    num_blocks = 8
    table = torch.arange(8, dtype=torch.int32).view(2, 4)
    table[1, 1] = 99                                    # logical block 1 of sequence 1
    paged = kvq.PagedKVCache(B, Hkv, cap, num_blocks, table.cuda())
    K, V = W.kv_batch(w, 0, 40, "cuda")
    sl = torch.zeros(B, dtype=torch.int32, device="cuda")
    gpu_append(paged, K, V, w, rt, sl)
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(paged) & kvq.KVQ_DEV_BAD_TABLE
    kvq.kvq_clear_status(paged)
    out = gpu_decode(paged, W.queries(w, "cuda"), w, rt, sl, 40)
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(paged) & kvq.KVQ_DEV_BAD_TABLE
    assert torch.isfinite(out[0]).all()


# --- values-only Hadamard rotation (the rotation split of "KVLinC", abstract) -------------------

@pytest.mark.parametrize("T", [37, 300])
def test_values_only_hadamard_rotation(T):
    """KVLinC rotates the values by a Hadamard matrix and leaves the keys
    unrotated (its key-error adapters are trained and not part of this
    library): the dense mode with R_k = I and R_v = H/sqrt(128) serves that
    split, through the CUDA-core (T=37) and tensor-core (T=300) appends."""
    import scipy.linalg
    B, Hkv, G = 2, 2, 2
    w = W.custom(seed=300 + T, B=B, Hq=Hkv * G, Hkv=Hkv, mode=0, k_outliers=6)
    Rk = np.stack([np.eye(D, dtype=np.float32)] * Hkv)
    Rv = np.stack([(scipy.linalg.hadamard(D) / np.sqrt(D)).astype(np.float32)] * Hkv)
    rt = (torch.from_numpy(Rk).cuda(), torch.from_numpy(Rv).cuda(), None)
    L0 = [0, 9]
    K = torch.stack([W.kv_rows(w, b, L0[b], L0[b] + T, "cpu")[0] for b in range(B)])
    V = torch.stack([W.kv_rows(w, b, L0[b], L0[b] + T, "cpu")[1] for b in range(B)])
    cap = ((max(L0) + T + 15) // 16) * 16
    cache = kvq.KVCache(B, Hkv, cap)
    sl = torch.tensor(L0, dtype=torch.int32, device="cuda")
    gpu_append(cache, K.cuda(), V.cuda(), w, rt, sl)
    oc = orc.Cache(B, Hkv, cap, 0)
    osl = np.array(L0, np.int32)
    assert orc.append(oc, f16bits(K), f16bits(V), 0, Rk, Rv, None, osl) == 0
    Q = W.queries(w, "cpu")
    ref, st = orc.decode(oc, f16bits(Q), 0, Rk, Rv, None, osl, n_threads=8)
    assert st == 0
    out = gpu_decode(cache, Q.cuda(), w, rt, sl, max(L0) + T)
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(cache) == 0
    err = rel_err(out.cpu().numpy(), ref)
    assert err.max() <= DEC_TOL, err.max()


def test_append_decode_step_equals_the_two_calls():
    """kvq_append_decode is the append followed by the decode: the same cache
    bytes, lengths and output bits; a call that fails its checks (workspace
    too small) enqueues nothing, the append included."""
    w = W.custom(seed=310, B=2, Hq=4, Hkv=2, mode=0, k_outliers=4)
    rt, _ = rot_tensors(w)
    cap, L0, T = 256, [100, 37], 1
    K = torch.stack([W.kv_rows(w, b, 0, 130, "cpu")[0] for b in range(2)]).cuda()
    V = torch.stack([W.kv_rows(w, b, 0, 130, "cpu")[1] for b in range(2)]).cuda()
    caches, outs, lens = [], [], []
    for fused in (False, True):
        cache = kvq.KVCache(2, 2, cap)
        sl = torch.zeros(2, dtype=torch.int32, device="cuda")
        gpu_append(cache, K[:, :100].contiguous(), V[:, :100].contiguous(), w, rt, sl)
        sl.copy_(torch.tensor(L0, dtype=torch.int32))
        Kn = K[:, 100:101].contiguous()
        Vn = V[:, 100:101].contiguous()
        Q = W.queries(w, "cuda")
        ws = kvq.decode_workspace(2, 4, 2, cap)
        out = torch.empty_like(Q)
        if fused:
            kvq.kvq_append_decode(Kn, Vn, Q, cache, 0, rt[0], rt[1], None, sl, cap, ws, out)
        else:
            gpu_append(cache, Kn, Vn, w, rt, sl)
            kvq.kvq_decode_attention(Q, cache, 0, rt[0], rt[1], None, sl, 0, cap, ws, out)
        torch.cuda.synchronize()
        assert kvq.kvq_get_status(cache) == 0
        caches.append(cache.blocks.clone())
        outs.append(out.clone())
        lens.append(sl.clone())
    assert torch.equal(caches[0], caches[1]) and torch.equal(outs[0], outs[1])
    assert torch.equal(lens[0], lens[1]) and list(lens[1].cpu().numpy()) == [101, 38]
    before = caches[1].clone()
    small = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_append_decode(Kn, Vn, Q, cache, 0, rt[0], rt[1], None, sl, cap, small, out)
    assert e.value.code == 5                               # KVQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.equal(cache.blocks, before) and list(sl.cpu().numpy()) == [101, 38]


@pytest.mark.parametrize("mode", [0, 1])
def test_append_decode_host_equals_the_device_step(mode):
    """kvq_append_decode_host is kvq_append_decode with its inputs and output
    in host memory: the same cache bytes, lengths and output bits; a call
    that fails its checks (workspace too small) touches neither the cache,
    the lengths nor the host output."""
    w = W.custom(seed=311 + mode, B=2, Hq=8, Hkv=2, mode=mode, k_outliers=4)
    rt, _ = rot_tensors(w)
    cap, L0, T = 256, [120, 53], 3
    K = torch.stack([W.kv_rows(w, b, 0, 140, "cpu")[0] for b in range(2)]).cuda()
    V = torch.stack([W.kv_rows(w, b, 0, 140, "cpu")[1] for b in range(2)]).cuda()
    Q = W.queries(w, "cuda")
    res = []
    for host in (False, True, "one buffer"):
        cache = kvq.KVCache(2, 2, cap, 4)
        sl = torch.zeros(2, dtype=torch.int32, device="cuda")
        gpu_append(cache, K[:, :120].contiguous(), V[:, :120].contiguous(), w, rt, sl)
        sl.copy_(torch.tensor(L0, dtype=torch.int32))
        Kn = K[:, 120:120 + T].contiguous()
        Vn = V[:, 120:120 + T].contiguous()
        if host:
            ws = kvq.step_workspace(2, T, 8, 2, cap)
            ws.fill_(0xFF)
            hO = torch.full(Q.shape, float("nan"), dtype=torch.float16).pin_memory()
            if host == "one buffer":          # back to back: a single H2D copy
                buf = torch.cat([Kn.reshape(-1), Vn.reshape(-1), Q.reshape(-1)]).cpu().pin_memory()
                n = Kn.numel()
                hk, hv = buf[:n].view(Kn.shape), buf[n:2 * n].view(Vn.shape)
                hq = buf[2 * n:].view(Q.shape)
            else:
                hk, hv, hq = Kn.cpu().pin_memory(), Vn.cpu().pin_memory(), Q.cpu().pin_memory()
            kvq.kvq_append_decode_host(hk, hv, hq, cache, mode, *rt, sl, cap, ws, hO)
            torch.cuda.synchronize()
            out = hO.cuda()
        else:
            ws = kvq.decode_workspace(2, 8, 2, cap)
            out = torch.empty_like(Q)
            kvq.kvq_append_decode(Kn, Vn, Q, cache, mode, *rt, sl, cap, ws, out)
            torch.cuda.synchronize()
        assert kvq.kvq_get_status(cache) == 0
        res.append((cache.blocks.clone(), cache.k_sink.clone(), out, sl.clone()))
    for r in res[1:]:
        for a, b in zip(res[0], r):
            assert torch.equal(a, b)
    assert list(res[1][3].cpu().numpy()) == [120 + T, 53 + T]
    before = cache.blocks.clone()
    small = torch.empty(64, dtype=torch.uint8, device="cuda")
    hO = torch.zeros(Q.shape, dtype=torch.float16).pin_memory()
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_append_decode_host(Kn.cpu().pin_memory(), Vn.cpu().pin_memory(),
                                   Q.cpu().pin_memory(), cache, mode, *rt, sl, cap, small, hO)
    assert e.value.code == 5                               # KVQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.equal(cache.blocks, before) and not hO.any()
    assert list(sl.cpu().numpy()) == [120 + T, 53 + T]


def test_append_decode_host_rejects_bad_calls():
    """Bad host-step calls fail before anything is enqueued: no rows (null
    input), a workspace off its 256-byte alignment, an output of the wrong
    shape, a device tensor where a host one belongs."""
    w = W.custom(seed=320, B=1, Hq=2, Hkv=2, mode=0)
    rt, _ = rot_tensors(w)
    cache = kvq.KVCache(1, 2, 64)
    sl = torch.zeros(1, dtype=torch.int32, device="cuda")
    Q = torch.zeros((1, 2, 128), dtype=torch.float16).pin_memory()
    hO = torch.zeros((1, 2, 128), dtype=torch.float16).pin_memory()
    ws = kvq.step_workspace(1, 1, 2, 2, 64)
    K0 = torch.zeros((1, 0, 2, 128), dtype=torch.float16)
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_append_decode_host(K0, K0, Q, cache, 0, *rt, sl, 64, ws, hO)
    assert e.value.code == 1                               # KVQ_ERR_INVALID_ARG
    K1 = torch.zeros((1, 1, 2, 128), dtype=torch.float16).pin_memory()
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_append_decode_host(K1, K1, Q, cache, 0, *rt, sl, 64, ws[16:], hO)
    assert e.value.code == 2                               # KVQ_ERR_UNSUPPORTED
    with pytest.raises(ValueError):
        kvq.kvq_append_decode_host(K1, K1, Q, cache, 0, *rt, sl, 64, ws, hO[:, :1])
    with pytest.raises(ValueError):
        kvq.kvq_append_decode_host(K1.cuda(), K1, Q, cache, 0, *rt, sl, 64, ws, hO)
    torch.cuda.synchronize()
    assert list(sl.cpu().numpy()) == [0] and kvq.kvq_get_status(cache) == 0


@pytest.mark.parametrize("layout", ["one buffer", "separate"])
def test_host_step_plan_equals_the_host_call(layout):
    """HostStep checks its arguments once and then runs kvq_append_decode_host
    with one C call per step: the same cache bytes, lengths and output bits as
    the plain call, also when each run names its own row of lengths; a
    lengths tensor of the wrong shape is refused."""
    w = W.custom(seed=330, B=2, Hq=4, Hkv=2, mode=0, k_outliers=4)
    rt, _ = rot_tensors(w)
    cap, T = 256, 2
    K = torch.stack([W.kv_rows(w, b, 0, 100, "cpu")[0] for b in range(2)])
    V = torch.stack([W.kv_rows(w, b, 0, 100, "cpu")[1] for b in range(2)])
    Q = W.queries(w, "cpu")
    res = []
    for use_plan in (False, True):
        cache = kvq.KVCache(2, 2, cap)
        sl = torch.zeros(2, dtype=torch.int32, device="cuda")
        gpu_append(cache, K[:, :90].contiguous().cuda(), V[:, :90].contiguous().cuda(), w, rt, sl)
        Kn, Vn = K[:, 90:90 + T].contiguous(), V[:, 90:90 + T].contiguous()
        if layout == "one buffer":     # views of one pinned buffer, as a serving loop keeps them
            buf = torch.cat([Kn.reshape(-1), Vn.reshape(-1), Q.reshape(-1)]).pin_memory()
            n = Kn.numel()
            hk, hv = buf[:n].view(Kn.shape), buf[n:2 * n].view(Vn.shape)
            hq = buf[2 * n:].view(Q.shape)
        else:                          # three pinned allocations (possibly adjacent)
            hk, hv, hq = Kn.pin_memory(), Vn.pin_memory(), Q.pin_memory()
        hO = torch.zeros(Q.shape, dtype=torch.float16).pin_memory()
        ws = kvq.step_workspace(2, T, 4, 2, cap)
        rows = torch.tensor([[90, 90], [92, 92]], dtype=torch.int32, device="cuda")
        outs = []
        plan = kvq.HostStep(hk, hv, hq, cache, 0, *rt, rows[0], cap, ws, hO) if use_plan else None
        for i in range(2):
            if use_plan:
                plan.run(rows[i])
            else:
                kvq.kvq_append_decode_host(hk, hv, hq, cache, 0, *rt, rows[i], cap, ws, hO)
            torch.cuda.synchronize()
            outs.append(hO.clone())
        assert kvq.kvq_get_status(cache) == 0
        res.append((cache.blocks.clone(), rows.clone(), outs))
        if use_plan:
            with pytest.raises(ValueError):
                plan.run(rows)                       # [2][2]: not int32 [B]
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])
    for a, b in zip(res[0][2], res[1][2]):
        assert torch.equal(a, b)
    assert list(res[1][1].cpu().numpy().ravel()) == [92, 92, 94, 94]
