"""Helpers shared by the GPU parity tests: run the same seeded inputs through
the CUDA path (libkvq) and through the CPU oracle, and compare."""
import numpy as np
import torch

import rotated_int2_kv_head_b200 as kvq
import workloads as W
from oracle import oracle as orc

D = 128


def f16bits(t):
    return W.f16_bits(t)


def rot_tensors(w, device="cuda"):
    Rk, Rv, perm = W.rotations(w)
    if w.mode == 0:
        return (torch.from_numpy(Rk).to(device), torch.from_numpy(Rv).to(device), None), (Rk, Rv, None)
    return (None, None, torch.from_numpy(perm).to(device)), (None, None, perm)


def append_variant(mode, T, B):
    """The rotation variant of kvq_debug_rotate_f32 that an append of T rows
    per sequence over B sequences runs (the library's documented size rule):
    1 = the tensor-core bulk kernel (dense: T >= 32, or T >= 8 with
    B*T >= 256; permutation + FWHT: T >= 128, or T >= 32 with B*T >= 1024),
    else 0."""
    if mode == 0:
        return 1 if T >= 32 or (T >= 8 and B * T >= 256) else 0
    return 1 if T >= 128 or (T >= 32 and B * T >= 1024) else 0


def gpu_append(cache, K, V, w, rt, seq_lens):
    kvq.kvq_rotate_quantize_append(K.contiguous(), V.contiguous(), w.mode, rt[0], rt[1], rt[2],
                                   cache, seq_lens)


def gpu_decode(cache, Q, w, rt, seq_lens, max_ctx):
    # The workspace need not be initialised: poison it (all bytes 0xFF, NaN
    # as fp32) so that a read of anything the call did not write shows up.
    ws = kvq.decode_workspace(cache.B, Q.shape[1], cache.Hkv, max_ctx)
    ws.fill_(0xFF)
    out = torch.empty_like(Q)
    kvq.kvq_decode_attention(Q.contiguous(), cache, w.mode, rt[0], rt[1], rt[2], seq_lens,
                             cache.sink_fp16, max_ctx, ws, out)
    return out


def upload_oracle_cache(oc, device="cuda"):
    """A libkvq cache holding the oracle's bytes (and its sink list)."""
    identified = oc.sink_pos is not None
    c = kvq.KVCache(oc.B, oc.Hkv, oc.capacity, oc.S, device=device, identified_sinks=identified)
    c.blocks.copy_(torch.from_numpy(oc.blocks.reshape(-1)))
    if oc.S > 0:
        c.k_sink.copy_(torch.from_numpy(oc.k_sink.view(np.float16)))
        c.v_sink.copy_(torch.from_numpy(oc.v_sink.view(np.float16)))
    if identified:
        c.sink_pos.copy_(torch.from_numpy(oc.sink_pos))
        c.sink_count.copy_(torch.from_numpy(oc.sink_count))
    return c


def download_cache(c):
    identified = getattr(c, "sink_pos", None) is not None
    oc = orc.Cache(c.B, c.Hkv, c.capacity, c.sink_fp16, identified=identified)
    oc.blocks[:] = c.block_view().cpu().numpy()
    if c.sink_fp16 > 0:
        oc.k_sink[:] = f16bits(c.k_sink)
        oc.v_sink[:] = f16bits(c.v_sink)
    if identified:
        oc.sink_pos[:] = c.sink_pos.cpu().numpy()
        oc.sink_count[:] = c.sink_count.cpu().numpy()
    return oc


def logical(oc, b, h, p):
    """(K codes[128], V codes[128], ks, kz, vs, vz) of position p."""
    kb, vb, ks, kz, vs, vz = orc.load_token(oc.blocks[b, h, p // 16], p % 16)
    return orc.unpack_row(kb), orc.unpack_row(vb), ks, kz, vs, vz


def rel_err(out_gpu, out_ref):
    """max-abs error / ||o_ref||_2 per (b, query head) row."""
    g = out_gpu.astype(np.float64).reshape(-1, D)
    r = out_ref.reshape(-1, D)
    return np.abs(g - r).max(axis=1) / np.maximum(np.linalg.norm(r, axis=1), 1e-30)


def near_tie_ok(x_rot_f64, codes_a, codes_b, s_bits, z_bits, tol=2e-3):
    """Every element where two code rows differ sits within tol of a rounding
    boundary of the grid (t = (x - z)/s close to k + 1/2)."""
    s = orc.f16_bits_to_f32(s_bits).astype(np.float64)
    z = orc.f16_bits_to_f32(z_bits).astype(np.float64)
    g = np.arange(D) // 32
    diff = np.nonzero(codes_a != codes_b)[0]
    for j in diff:
        if s[g[j]] == 0:
            return False
        t = (x_rot_f64[j] - z[g[j]]) / s[g[j]]
        if abs((t - 0.5) - np.round(t - 0.5)) > tol:
            return False
    return True
