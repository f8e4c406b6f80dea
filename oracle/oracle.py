"""numpy front end of the C oracle (kvq_oracle.c).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).  Arrays are passed to C as
raw pointers; every function copies its inputs to contiguous arrays of the
exact dtype the C side expects.  Cache buffers use the library's byte format
(blocks of 16 tokens, 1536 bytes), so results can be compared byte for byte.
"""
import ctypes as C

import numpy as np

from . import build as _build

D = 128
NG = 4
BLK_TOK = 16
BLK_BYTES = 1536
ST_CAPACITY = 1
ST_BAD_LEN = 2

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        p = C.c_void_p
        i64 = C.c_int64
        ci = C.c_int
        L.orc_f32_to_f16.restype = C.c_uint16
        L.orc_f32_to_f16.argtypes = [C.c_float]
        L.orc_f16_to_f32.restype = C.c_float
        L.orc_f16_to_f32.argtypes = [C.c_uint16]
        L.orc_f32_to_f16_array.argtypes = [p, i64, p]
        L.orc_f16_to_f32_array.argtypes = [p, i64, p]
        L.orc_fwht_f64.argtypes = [p, ci]
        L.orc_rotate_f64_rows.argtypes = [p, i64, ci, p, p, p]
        L.orc_unrotate_f64_rows.argtypes = [p, i64, ci, p, p, p]
        L.orc_rotate_rows_f32.argtypes = [p, i64, ci, p, p, p]
        L.orc_quantize_rows.argtypes = [p, i64, p, p, p]
        L.orc_pack_row.argtypes = [p, p]
        L.orc_unpack_row.argtypes = [p, p]
        L.orc_store_token.argtypes = [p, ci, p, p, p, p, p, p]
        L.orc_load_token.argtypes = [p, ci, p, p, p, p, p, p]
        L.orc_identify_sinks.argtypes = [p, ci, ci, C.c_float, ci, ci, p, p, p]
        L.orc_append.restype = ci
        L.orc_append.argtypes = [p, p, ci, ci, ci, ci, p, p, p, ci, ci, p, p, p, p, p, p]
        L.orc_decode.restype = ci
        L.orc_decode.argtypes = [p, ci, ci, ci, ci, p, p, p, ci, ci, p, p, p, p, p, p, ci, ci,
                                 ci, p]
        L.orc_decode_adapter.restype = ci
        L.orc_decode_adapter.argtypes = [p, ci, ci, ci, ci, p, p, p, ci, ci, p, p, p, p, p, p, p, p,
                                         ci, ci, p]
        L.orc_attention_f64.argtypes = [p, p, p, ci, p]
        L.orc_rope_f64.argtypes = [p, i64, C.c_double]
        L.orc_rotate_group_f64.argtypes = [p, ci, p, p]
        L.orc_unrotate_group_f64.argtypes = [p, ci, p, p]
        L.orc_append_prerope.restype = ci
        L.orc_append_prerope.argtypes = [p, p, ci, ci, ci, ci, p, ci, ci, p, p, p, p, p, p]
        L.orc_decode_prerope.restype = ci
        L.orc_decode_prerope.argtypes = [p, ci, ci, ci, ci, p, C.c_double, ci, ci, p, p, p, p, p, p,
                                         ci, ci, ci, p]
        _lib = L
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


# --- binary16 ------------------------------------------------------------------

def f32_to_f16_bits(x):
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().orc_f32_to_f16_array(_p(x), x.size, _p(out))
    return out


def f16_bits_to_f32(h):
    h = _c(h, np.uint16)
    out = np.empty(h.shape, np.float32)
    lib().orc_f16_to_f32_array(_p(h), h.size, _p(out))
    return out


# --- rotations -------------------------------------------------------------------

def fwht_f64(y):
    y = _c(y, np.float64).copy()
    lib().orc_fwht_f64(_p(y), y.shape[-1])
    return y


def _rot_args(mode, R, perm):
    Rc = _c(R, np.float32) if mode == 0 else None
    pc = _c(perm, np.int32) if mode == 1 else None
    return Rc, pc


def rotate_f64(x, mode, R=None, perm=None):
    """fp64 rows x [n,128] -> x.R (dense) or FWHT(x[perm])/sqrt(128)."""
    x = _c(x, np.float64).reshape(-1, D)
    Rc, pc = _rot_args(mode, R, perm)
    out = np.empty_like(x)
    lib().orc_rotate_f64_rows(_p(x), x.shape[0], mode, _p(Rc), _p(pc), _p(out))
    return out


def unrotate_f64(o, mode, R=None, perm=None):
    o = _c(o, np.float64).reshape(-1, D)
    Rc, pc = _rot_args(mode, R, perm)
    out = np.empty_like(o)
    lib().orc_unrotate_f64_rows(_p(o), o.shape[0], mode, _p(Rc), _p(pc), _p(out))
    return out


def rotate_rows_f32(x_f16bits, mode, R=None, perm=None):
    """fp16 rows (as uint16 bit patterns) [n,128] -> rotated fp32 rows."""
    x = _c(x_f16bits, np.uint16).reshape(-1, D)
    Rc, pc = _rot_args(mode, R, perm)
    out = np.empty(x.shape, np.float32)
    lib().orc_rotate_rows_f32(_p(x), x.shape[0], mode, _p(Rc), _p(pc), _p(out))
    return out


# --- quantizer / packing -------------------------------------------------------------

def quantize_rows(x):
    """fp32 rows [n,128] -> (codes u8 [n,128], s u16 [n,4], z u16 [n,4])."""
    x = _c(x, np.float32).reshape(-1, D)
    n = x.shape[0]
    codes = np.empty((n, D), np.uint8)
    s = np.empty((n, NG), np.uint16)
    z = np.empty((n, NG), np.uint16)
    lib().orc_quantize_rows(_p(x), n, _p(codes), _p(s), _p(z))
    return codes, s, z


def pack_row(codes):
    codes = _c(codes, np.uint8)
    out = np.empty(32, np.uint8)
    lib().orc_pack_row(_p(codes), _p(out))
    return out


def unpack_row(b):
    b = _c(b, np.uint8)
    out = np.empty(D, np.uint8)
    lib().orc_unpack_row(_p(b), _p(out))
    return out


def store_token(block, tau, kbytes, vbytes, ks, kz, vs, vz):
    assert block.dtype == np.uint8 and block.flags.c_contiguous and block.size >= BLK_BYTES
    args = [_c(a, t) for a, t in ((kbytes, np.uint8), (vbytes, np.uint8), (ks, np.uint16),
                                  (kz, np.uint16), (vs, np.uint16), (vz, np.uint16))]
    lib().orc_store_token(_p(block), tau, *[_p(a) for a in args])


def load_token(block, tau):
    block = _c(block, np.uint8)
    kb = np.empty(32, np.uint8)
    vb = np.empty(32, np.uint8)
    ks, kz, vs, vz = (np.empty(NG, np.uint16) for _ in range(4))
    lib().orc_load_token(_p(block), tau, _p(kb), _p(vb), _p(ks), _p(kz), _p(vs), _p(vz))
    return kb, vb, ks, kz, vs, vz


# --- cache ---------------------------------------------------------------------------

class Cache:
    """Host copy of a packed cache in the library's byte format.
    identified=True: sinks are the positions identify_sinks picks (listed in
    sink_pos [B][S], sink_count [B]); otherwise the leading S positions."""

    def __init__(self, B, Hkv, capacity, S, identified=False):
        assert capacity % BLK_TOK == 0
        assert not identified or S >= 1
        self.B, self.Hkv, self.capacity, self.S = B, Hkv, capacity, S
        self.blocks = np.zeros((B, Hkv, capacity // BLK_TOK, BLK_BYTES), np.uint8)
        self.k_sink = np.zeros((B, Hkv, max(S, 0), D), np.uint16)
        self.v_sink = np.zeros((B, Hkv, max(S, 0), D), np.uint16)
        self.sink_pos = np.zeros((B, S), np.int32) if identified else None
        self.sink_count = np.zeros(B, np.int32) if identified else None


def identify_sinks(cache, act, tau, seq_lens):
    """act: fp32 [B][T] activation magnitudes of the next T tokens.  Adds
    the picked positions to cache.sink_pos / sink_count (in place)."""
    assert cache.sink_pos is not None
    act = _c(act, np.float32)
    B, T = act.shape
    sl = _c(seq_lens, np.int32)
    lib().orc_identify_sinks(_p(act), B, T, float(tau), cache.S, cache.capacity, _p(sl),
                             _p(cache.sink_pos), _p(cache.sink_count))


def append(cache, K, V, mode, R_k=None, R_v=None, perm=None, seq_lens=None):
    """K, V: fp16 bit patterns [B][T][Hkv][128].  Updates cache and seq_lens
    (int32 [B], in place).  Returns the status bits."""
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    B, T, Hkv, d = K.shape
    assert d == D and B == cache.B and Hkv == cache.Hkv and V.shape == K.shape
    assert seq_lens.dtype == np.int32 and seq_lens.flags.c_contiguous
    Rk = _c(R_k, np.float32) if mode == 0 else None
    Rv = _c(R_v, np.float32) if mode == 0 else None
    pc = _c(perm, np.int32) if mode == 1 else None
    return lib().orc_append(_p(K), _p(V), B, T, Hkv, mode, _p(Rk), _p(Rv), _p(pc),
                            cache.capacity, cache.S, _p(cache.blocks), _p(cache.k_sink),
                            _p(cache.v_sink), _p(seq_lens), _p(cache.sink_pos),
                            _p(cache.sink_count))


def decode(cache, Q, mode, R_k=None, R_v=None, perm=None, seq_lens=None,
           only_b=-1, only_h=-1, n_threads=1):
    """Q: fp16 bit patterns [B][Hq][128].  Returns (out fp64 [B][Hq][128],
    status).  only_b / only_h restrict the work to one sequence / KV head."""
    Q = _c(Q, np.uint16)
    B, Hq, d = Q.shape
    assert d == D and B == cache.B and Hq % cache.Hkv == 0
    Rk = _c(R_k, np.float32) if mode == 0 else None
    Rv = _c(R_v, np.float32) if mode == 0 else None
    pc = _c(perm, np.int32) if mode == 1 else None
    sl = _c(seq_lens, np.int32)
    out = np.zeros((B, Hq, D), np.float64)
    st = lib().orc_decode(_p(Q), B, Hq, cache.Hkv, mode, _p(Rk), _p(Rv), _p(pc),
                          cache.capacity, cache.S, _p(cache.blocks), _p(cache.k_sink),
                          _p(cache.v_sink), _p(sl), _p(cache.sink_pos), _p(cache.sink_count),
                          only_b, only_h, n_threads, _p(out))
    return out, st


def decode_adapter(cache, Q, mode, R_k, R_v, perm, seq_lens, U, V, n_threads=1):
    """decode with KVLinC key correction adapters: U, V fp32 [Hkv][128][r];
    every INT2 key k^ (model basis) is scored as k^ + (k^ . U) . V^T.
    Returns (out fp64 [B][Hq][128], status)."""
    Q = _c(Q, np.uint16)
    B, Hq, d = Q.shape
    assert d == D and B == cache.B and Hq % cache.Hkv == 0
    Rk = _c(R_k, np.float32) if mode == 0 else None
    Rv = _c(R_v, np.float32) if mode == 0 else None
    pc = _c(perm, np.int32) if mode == 1 else None
    U = _c(U, np.float32)
    V = _c(V, np.float32)
    assert U.shape == V.shape and U.shape[:2] == (cache.Hkv, D)
    r = U.shape[2]
    sl = _c(seq_lens, np.int32)
    out = np.zeros((B, Hq, D), np.float64)
    st = lib().orc_decode_adapter(_p(Q), B, Hq, cache.Hkv, mode, _p(Rk), _p(Rv), _p(pc),
                                  cache.capacity, cache.S, _p(cache.blocks), _p(cache.k_sink),
                                  _p(cache.v_sink), _p(sl), _p(cache.sink_pos),
                                  _p(cache.sink_count), _p(U), _p(V), r, n_threads, _p(out))
    return out, st


def attention_f64(q, K, V):
    q = _c(q, np.float64)
    K = _c(K, np.float64).reshape(-1, D)
    V = _c(V, np.float64).reshape(-1, D)
    out = np.empty(D, np.float64)
    lib().orc_attention_f64(_p(q), _p(K), _p(V), K.shape[0], _p(out))
    return out


# --- pre-RoPE grouped-head rotation (keys rotated before RoPE, across gh heads) ----------

def rope_f64(x, t, base):
    """RoPE (rotate-half pairing) of one fp64 row x [128] at position t."""
    x = _c(x, np.float64).copy()
    lib().orc_rope_f64(_p(x), int(t), float(base))
    return x


def rotate_group_f64(x, perm):
    """x [n] -> FWHT_n(x[perm]) / sqrt(n)."""
    x = _c(x, np.float64)
    pc = _c(perm, np.int32)
    out = np.empty_like(x)
    lib().orc_rotate_group_f64(_p(x), x.size, _p(pc), _p(out))
    return out


def unrotate_group_f64(o, perm):
    o = _c(o, np.float64)
    pc = _c(perm, np.int32)
    out = np.empty_like(o)
    lib().orc_unrotate_group_f64(_p(o), o.size, _p(pc), _p(out))
    return out


def append_prerope(cache, K, V, gh, perm, seq_lens):
    """K (pre-RoPE), V: fp16 bit patterns [B][T][Hkv][128]; perm int32
    [2][Hkv*128] (plane 0: Hkv/gh key permutations of 128*gh entries; plane 1:
    one value permutation of 128 per head).  Sinks (leading or identified) keep
    the pre-RoPE key as given and the rotated value, in fp16."""
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    B, T, Hkv, d = K.shape
    assert d == D and B == cache.B and Hkv == cache.Hkv and V.shape == K.shape and Hkv % gh == 0
    assert seq_lens.dtype == np.int32 and seq_lens.flags.c_contiguous
    pc = _c(perm, np.int32).reshape(2, Hkv * D)
    return lib().orc_append_prerope(_p(K), _p(V), B, T, Hkv, gh, _p(pc), cache.capacity, cache.S,
                                    _p(cache.blocks), _p(cache.k_sink), _p(cache.v_sink),
                                    _p(seq_lens), _p(cache.sink_pos), _p(cache.sink_count))


def decode_prerope(cache, Q, gh, perm, rope_base, seq_lens, only_b=-1, only_h=-1, n_threads=1):
    """Q: fp16 bit patterns [B][Hq][128] (post-RoPE).  Returns (out fp64, status)."""
    Q = _c(Q, np.uint16)
    B, Hq, d = Q.shape
    assert d == D and B == cache.B and Hq % cache.Hkv == 0
    pc = _c(perm, np.int32).reshape(2, cache.Hkv * D)
    sl = _c(seq_lens, np.int32)
    out = np.zeros((B, Hq, D), np.float64)
    st = lib().orc_decode_prerope(_p(Q), B, Hq, cache.Hkv, gh, _p(pc), float(rope_base),
                                  cache.capacity, cache.S, _p(cache.blocks), _p(cache.k_sink),
                                  _p(cache.v_sink), _p(sl), _p(cache.sink_pos),
                                  _p(cache.sink_count), only_b, only_h, n_threads, _p(out))
    return out, st
