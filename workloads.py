"""Seeded synthetic workloads for the rotated INT2 KV-cache hot path.

This module only draws inputs; it holds none of the method's arithmetic.
Both the CUDA path (through the library) and the CPU oracle consume the very
same tensors drawn here.

The five workloads (head_dim 128, INT2 groups of 32 along head_dim):
  tiny        B=1, 1 head, context 4096, dense rotation, 4 key outlier
              channels x20, no sinks.
  llama7b     B=1, 32 heads (MHA), context 32768 = 32767 prefilled + 1
              appended, 8 key outlier channels x20 per head, dense rotation.
  hadamard    B=16, 32 heads, context 8192 = 8064 prefilled + a 128-token
              chunk appended, per-channel scales log-uniform in [0.5, 20]
              on K and V, channel permutation + FWHT rotation.
  gqa_sinks   B=8, 32 query heads over 8 KV heads, context 131072, first 4
              tokens kept fp16 (sinks), sink keys x50, dense rotation.
  ragged      B=64, 32 heads, context lengths uniform in [1024, 65536],
              dense rotation, 8 key outlier channels x20; plus a separate
              bulk append of 32768 prefill tokens x 32 heads for B=4.
  gqa8        B=4, 64 query heads over 8 KV heads (G = 8), context 65536,
              dense rotation, 8 key outlier channels x20.
  ragged_b8   the first 8 sequences of ragged (for profiler captures).
  gqa_sinks_identified
              gqa_sinks, but the 4 fp16 rows go to the tokens picked by their
              activation magnitude: position 0 and each other token with
              probability 4e-5 are massive (magnitude >= 1000, keys x50).

Every K/V row is drawn from a stream keyed by (workload, kind, sequence,
1024-token chunk), so any token range can be regenerated on its own without
drawing the rest.  The stream depends on the device it is drawn on (torch's
CPU and CUDA generators differ): a comparison draws once, on one device, and
hands the same tensor to both sides.
"""
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

D = 128
CHUNK = 1024


@dataclass
class Workload:
    name: str
    seed: int
    B: int
    Hq: int
    Hkv: int
    mode: int                    # 0 dense rotation, 1 permutation + FWHT
    sink: int = 0
    context: int = 0             # decode context per sequence (uniform case)
    append_T: int = 1            # tokens appended by the step before decode
    k_outliers: int = 0          # key channels scaled by outlier_scale
    outlier_scale: float = 20.0
    channel_scale: Optional[tuple] = None   # (lo, hi) log-uniform per channel
    sink_key_scale: float = 1.0
    ragged: Optional[tuple] = None          # (lo, hi) uniform context lengths
    # identified sinks: each token is "massive" with this probability (and
    # position 0 always is); its activation magnitude is >= 1000 against
    # |N(0,1)| for the rest, and its key row is scaled by sink_key_scale
    massive_rate: float = 0.0
    extra: dict = field(default_factory=dict)

    @property
    def G(self):
        return self.Hq // self.Hkv

    def seq_lens(self) -> np.ndarray:
        """Decode context per sequence (including the appended tokens)."""
        if self.ragged is None:
            return np.full(self.B, self.context, np.int64)
        rng = np.random.default_rng([self.seed, 7])
        lo, hi = self.ragged
        return rng.integers(lo, hi + 1, size=self.B)

    def capacity(self) -> int:
        return int(-(-int(self.seq_lens().max()) // 16) * 16)


WORKLOADS = {
    "tiny": Workload("tiny", 1001, B=1, Hq=1, Hkv=1, mode=0, context=4096, k_outliers=4),
    "llama7b": Workload("llama7b", 1002, B=1, Hq=32, Hkv=32, mode=0, context=32768,
                        append_T=1, k_outliers=8),
    "hadamard": Workload("hadamard", 1003, B=16, Hq=32, Hkv=32, mode=1, context=8192,
                         append_T=128, channel_scale=(0.5, 20.0)),
    "gqa_sinks": Workload("gqa_sinks", 1004, B=8, Hq=32, Hkv=8, mode=0, sink=4,
                          context=131072, sink_key_scale=50.0),
    "ragged": Workload("ragged", 1005, B=64, Hq=32, Hkv=32, mode=0, ragged=(1024, 65536),
                       k_outliers=8, extra={"prefill_B": 4, "prefill_T": 32768}),
    # eight query heads per KV head (64 over 8), the widest GQA grouping the
    # library takes
    "gqa8": Workload("gqa8", 1007, B=4, Hq=64, Hkv=8, mode=0, context=65536, k_outliers=8),
    # the first 8 sequences of ragged (same seed, so the same lengths): a
    # cache of 1.6 GB, small enough for a full profiler capture of the
    # decode kernels, whose counters scale to ragged by the bytes read
    "ragged_b8": Workload("ragged_b8", 1005, B=8, Hq=32, Hkv=32, mode=0, ragged=(1024, 65536),
                          k_outliers=8),
    # gqa_sinks with its 4 fp16 rows given to the massive tokens instead of
    # the leading ones (position 0 plus about 5 more per sequence)
    "gqa_sinks_identified": Workload("gqa_sinks_identified", 1006, B=8, Hq=32, Hkv=8, mode=0,
                                     sink=4, context=131072, sink_key_scale=50.0,
                                     massive_rate=4e-5),
}

# activation magnitude at and above which a token counts as massive (the
# drawn magnitudes are |N(0,1)| or >= 1000)
MASSIVE_TAU = 100.0


def custom(name="custom", seed=1, B=1, Hq=1, Hkv=1, mode=0, sink=0, context=64,
           append_T=1, k_outliers=0, channel_scale=None, sink_key_scale=1.0, massive_rate=0.0,
           ragged=None) -> Workload:
    """A small workload of the same families, for edge-case tests."""
    return Workload(name, seed, B=B, Hq=Hq, Hkv=Hkv, mode=mode, sink=sink, context=context,
                    append_T=append_T, k_outliers=k_outliers, channel_scale=channel_scale,
                    sink_key_scale=sink_key_scale, ragged=ragged, massive_rate=massive_rate)


# --- rotations and per-channel structure (numpy, seeded) -------------------------------

def random_orthogonal(rng, n=D) -> np.ndarray:
    """Haar-random orthogonal matrix: QR of a Gaussian, signs fixed by diag(R)."""
    a = rng.standard_normal((n, n))
    q, r = np.linalg.qr(a)
    q *= np.sign(np.diag(r))[None, :]
    return q


def rotations(w: Workload):
    """Dense mode: (R_k, R_v) fp32 [Hkv][128][128].  FWHT mode: perm int32
    [2][Hkv][128] (plane 0 keys, plane 1 values).  Returns (R_k, R_v, perm)."""
    rng = np.random.default_rng([w.seed, 11])
    if w.mode == 0:
        Rk = np.stack([random_orthogonal(rng) for _ in range(w.Hkv)]).astype(np.float32)
        Rv = np.stack([random_orthogonal(rng) for _ in range(w.Hkv)]).astype(np.float32)
        return Rk, Rv, None
    perm = np.stack([np.stack([rng.permutation(D) for _ in range(w.Hkv)]) for _ in range(2)])
    return None, None, perm.astype(np.int32)


def channel_scales(w: Workload):
    """Per (KV head, channel) multipliers for K and for V, fp32 [Hkv][128]."""
    rng = np.random.default_rng([w.seed, 13])
    ks = np.ones((w.Hkv, D), np.float32)
    vs = np.ones((w.Hkv, D), np.float32)
    if w.k_outliers:
        for h in range(w.Hkv):
            ks[h, rng.choice(D, w.k_outliers, replace=False)] = w.outlier_scale
    if w.channel_scale is not None:
        lo, hi = np.log(w.channel_scale[0]), np.log(w.channel_scale[1])
        ks *= np.exp(rng.uniform(lo, hi, size=(w.Hkv, D))).astype(np.float32)
        vs *= np.exp(rng.uniform(lo, hi, size=(w.Hkv, D))).astype(np.float32)
    return ks, vs


# --- K / V rows and queries (torch, any device) ----------------------------------------

def _chunk_rows(w: Workload, kind: int, b: int, chunk: int, device) -> torch.Tensor:
    g = torch.Generator(device=device)
    key = ((w.seed * 1_000_003 + kind) * 1_000_033 + b) * 1_000_037 + chunk
    g.manual_seed(key % (1 << 62))
    return torch.randn((CHUNK, w.Hkv, D), generator=g, device=device, dtype=torch.float32)


def _chunk_act(w: Workload, b: int, chunk: int) -> np.ndarray:
    rng = np.random.default_rng([w.seed, 77, b, chunk])
    a = np.abs(rng.standard_normal(CHUNK)).astype(np.float32)
    massive = rng.random(CHUNK) < w.massive_rate
    if chunk == 0:
        massive[0] = True
    a[massive] = (1000.0 * (1.0 + rng.random(int(massive.sum())))).astype(np.float32)
    return a


def activations(w: Workload, b: int, t0: int, t1: int) -> np.ndarray:
    """Activation magnitude of the tokens [t0, t1) of sequence b, fp32 (numpy):
    |N(0,1)|, or >= 1000 for massive tokens (none unless massive_rate > 0)."""
    if t1 <= t0:
        return np.zeros(0, np.float32)
    if w.massive_rate <= 0.0:
        return np.abs(np.random.default_rng([w.seed, 78, b, t0]).standard_normal(t1 - t0)
                      ).astype(np.float32)
    parts = [_chunk_act(w, b, c) for c in range(t0 // CHUNK, (t1 - 1) // CHUNK + 1)]
    a = np.concatenate(parts)
    return a[t0 - (t0 // CHUNK) * CHUNK:][:t1 - t0]


def kv_rows(w: Workload, b: int, t0: int, t1: int, device="cpu"):
    """K and V rows of sequence b for positions [t0, t1): fp16 [t1-t0][Hkv][128]."""
    ks, vs = channel_scales(w)
    kt = torch.from_numpy(ks).to(device)
    vt = torch.from_numpy(vs).to(device)
    outs = []
    for kind, sc in ((0, kt), (1, vt)):
        parts = []
        for c in range(t0 // CHUNK, (t1 - 1) // CHUNK + 1 if t1 > t0 else t0 // CHUNK):
            rows = _chunk_rows(w, kind, b, c, device)
            lo = max(t0, c * CHUNK) - c * CHUNK
            hi = min(t1, (c + 1) * CHUNK) - c * CHUNK
            parts.append(rows[lo:hi])
        x = torch.cat(parts) if parts else torch.empty((0, w.Hkv, D), device=device)
        x = x * sc[None]
        if w.massive_rate > 0.0:
            if kind == 0 and w.sink_key_scale != 1.0 and t1 > t0:
                m = torch.from_numpy(activations(w, b, t0, t1) >= MASSIVE_TAU).to(device)
                x[m] *= w.sink_key_scale
        elif kind == 0 and w.sink and w.sink_key_scale != 1.0 and t0 < w.sink:
            n = min(w.sink, t1) - t0
            x[:n] *= w.sink_key_scale
        outs.append(x.to(torch.float16))
    return outs[0], outs[1]


def kv_batch(w: Workload, t0: int, t1: int, device="cpu", bs=None):
    """K, V fp16 [B'][t1-t0][Hkv][128] for sequences bs (default all)."""
    bs = range(w.B) if bs is None else bs
    ks, vs = zip(*(kv_rows(w, b, t0, t1, device) for b in bs))
    return torch.stack(ks), torch.stack(vs)


def queries(w: Workload, device="cpu", step: int = 0) -> torch.Tensor:
    """Decode queries fp16 [B][Hq][128], N(0,1)."""
    g = torch.Generator(device=device)
    g.manual_seed(w.seed * 7919 + 17 + step)
    return torch.randn((w.B, w.Hq, D), generator=g, device=device).to(torch.float16)


def f16_bits(t: torch.Tensor) -> np.ndarray:
    """fp16 tensor -> numpy uint16 bit patterns (host)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


# --- pre-RoPE grouped-head rotation -------------------------------------------------------

def prerope_perm(w: Workload, gh: int) -> np.ndarray:
    """int32 [2][Hkv*128]: plane 0 the Hkv/gh key-group permutations of
    128*gh channels, plane 1 one value permutation of 128 per head (seeded)."""
    rng = np.random.default_rng([w.seed, 91, gh])
    keys = np.concatenate([rng.permutation(D * gh) for _ in range(w.Hkv // gh)])
    vals = np.concatenate([rng.permutation(D) for _ in range(w.Hkv)])
    return np.stack([keys, vals]).astype(np.int32)
