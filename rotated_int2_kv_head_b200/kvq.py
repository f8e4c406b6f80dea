"""Thin Python binding of libkvq's C ABI (include/kvq.h).

Argument marshalling only: torch tensors are checked for dtype, shape and
contiguity and passed to the library as raw device pointers together with
the current CUDA stream.  Every step of the computation runs in libkvq's
CUDA kernels; there is no Python or CPU fallback.  If libkvq.so is missing
the import fails with an error that says how to build it.
"""
import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

D = 128
GROUP = 32
BLOCK_TOKENS = 16
BLOCK_BYTES = 1536

KVQ_ROT_DENSE = 0
KVQ_ROT_PERM_FWHT = 1

KVQ_DEV_CAPACITY = 1
KVQ_DEV_BAD_LEN = 2
KVQ_DEV_TIMEOUT = 4
KVQ_DEV_BAD_TABLE = 8

_STATUS = {0: "KVQ_OK", 1: "KVQ_ERR_INVALID_ARG", 2: "KVQ_ERR_UNSUPPORTED", 3: "KVQ_ERR_CUDA",
           4: "KVQ_ERR_CAPACITY", 5: "KVQ_ERR_WORKSPACE"}


class KvqError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__("%s failed: %s (%d)" % (fn, _STATUS.get(code, "?"), code))
        self.code = code


class CacheDesc(C.Structure):
    _fields_ = [("B", C.c_int32), ("Hkv", C.c_int32), ("head_dim", C.c_int32),
                ("group", C.c_int32), ("capacity", C.c_int32), ("sink_fp16", C.c_int32),
                ("blocks", C.c_void_p), ("k_sink", C.c_void_p), ("v_sink", C.c_void_p),
                ("status", C.c_void_p), ("block_table", C.c_void_p), ("num_blocks", C.c_int32),
                ("sink_pos", C.c_void_p), ("sink_count", C.c_void_p)]


_lib = None


def lib():
    """Load libkvq.so (built in-tree by rotated_int2_kv_head_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError("libkvq.so is not built (%s); run `python -m "
                          "rotated_int2_kv_head_b200.build`" % LIB_PATH)
    L = C.CDLL(LIB_PATH)
    p, i32, sz = C.c_void_p, C.c_int32, C.c_size_t
    L.kvq_cache_bytes.restype = sz
    L.kvq_cache_bytes.argtypes = [i32, i32, i32]
    L.kvq_rotate_quantize_append.restype = C.c_int
    L.kvq_rotate_quantize_append.argtypes = [p, p, i32, C.c_int, p, p, p, C.POINTER(CacheDesc), p, p]
    L.kvq_identify_sinks.restype = C.c_int
    L.kvq_identify_sinks.argtypes = [p, i32, C.c_float, C.POINTER(CacheDesc), p, p]
    L.kvq_append_decode.restype = C.c_int
    L.kvq_append_decode.argtypes = [p, p, i32, p, i32, C.POINTER(CacheDesc), C.c_int, p, p, p, p,
                                    i32, p, sz, p, p]
    L.kvq_step_workspace_size.restype = sz
    L.kvq_step_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32]
    L.kvq_append_decode_host.restype = C.c_int
    L.kvq_append_decode_host.argtypes = [p, p, i32, p, i32, C.POINTER(CacheDesc), C.c_int, p, p,
                                         p, p, i32, p, sz, p, p]
    L.kvq_prerope_append.restype = C.c_int
    L.kvq_prerope_append.argtypes = [p, p, i32, i32, p, C.POINTER(CacheDesc), p, p]
    L.kvq_prerope_workspace_size.restype = sz
    L.kvq_prerope_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32]
    L.kvq_prerope_decode.restype = C.c_int
    L.kvq_prerope_decode.argtypes = [p, i32, C.POINTER(CacheDesc), i32, p, C.c_float, p, i32, p,
                                     sz, p, p]
    L.kvq_debug_rotate_group_f32.restype = C.c_int
    L.kvq_debug_rotate_group_f32.argtypes = [p, i32, i32, p, p, p]
    L.kvq_decode_workspace_size.restype = sz
    L.kvq_decode_workspace_size.argtypes = [i32, i32, i32, i32, i32]
    L.kvq_decode_attention.restype = C.c_int
    L.kvq_decode_attention.argtypes = [p, i32, C.POINTER(CacheDesc), C.c_int, p, p, p, p, i32, i32,
                                       p, sz, p, p]
    L.kvq_decode_attention_timed.restype = C.c_int
    L.kvq_decode_attention_timed.argtypes = [p, i32, C.POINTER(CacheDesc), C.c_int, p, p, p, p, i32,
                                             i32, p, sz, p, p, p, p]
    L.kvq_decode_attention_ex.restype = C.c_int
    L.kvq_decode_attention_ex.argtypes = [p, i32, i32, C.c_uint32, C.POINTER(CacheDesc), C.c_int, p,
                                          p, p, p, i32, i32, p, sz, p, p]
    L.kvq_decode_attention_adapter.restype = C.c_int
    L.kvq_decode_attention_adapter.argtypes = [p, i32, i32, C.c_uint32, C.POINTER(CacheDesc),
                                               C.c_int, p, p, p, p, p, i32, p, i32, i32, p, sz, p,
                                               p]
    L.kvq_decode_attention_noalloc.restype = C.c_int
    L.kvq_decode_attention_noalloc.argtypes = [p, i32, C.POINTER(CacheDesc), C.c_int, p, p, p, p,
                                               i32, i32, p, p]
    L.kvq_get_status.restype = C.c_int
    L.kvq_get_status.argtypes = [C.POINTER(CacheDesc), p, C.POINTER(C.c_int32)]
    L.kvq_clear_status.restype = C.c_int
    L.kvq_clear_status.argtypes = [C.POINTER(CacheDesc), p]
    L.kvq_debug_rotate_f32.restype = C.c_int
    L.kvq_debug_rotate_f32.argtypes = [p, i32, C.c_int, p, p, i32, p, p]
    L.kvq_debug_quantize_f32.restype = C.c_int
    L.kvq_debug_quantize_f32.argtypes = [p, i32, p, p, p]
    L.kvq_debug_wait_timeout.restype = C.c_int
    L.kvq_debug_wait_timeout.argtypes = [p, C.c_uint32, p, p, p]
    L.kvq_status_string.restype = C.c_char_p
    L.kvq_status_string.argtypes = [C.c_int]
    _lib = L
    return L


def _ptr(t):
    # ctypes turns the int into the c_void_p argument
    return None if t is None else t.data_ptr()


# torch's raw current-stream query (an int, no Stream object); the public
# torch.cuda.current_stream() builds a Python object per call, which costs
# more than a kernel launch on the host.  Fall back to it if absent.
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream, t=None):
    """cudaStream_t (as an int) for a call on tensor t's device: `stream` if
    given, else torch's current stream of that device."""
    if stream is not None:
        return stream.cuda_stream
    if _raw_stream is not None and t is not None:
        return _raw_stream(t.get_device())
    return torch.cuda.current_stream().cuda_stream


def _check(fn, code):
    if code != 0:
        raise KvqError(fn, code)


def _need_shape(t, dtype, name, shape=None):
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if shape is not None and t.shape != shape:
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))


def _need(t, dtype, name, shape=None):
    if t is None:
        return
    _need_shape(t, dtype, name, shape)
    if not (t.is_cuda and t.is_contiguous()):
        raise ValueError("%s must be a contiguous CUDA tensor" % name)


def _need_rotation(mode, R_k, R_v, perm, Hkv):
    """The rotation inputs of `mode`: dense R_k, R_v fp32 [Hkv][128][128], or
    perm int32 [2][Hkv][128].  The C ABI cannot see their sizes, so an
    undersized tensor would be read out of bounds on the device."""
    if mode == KVQ_ROT_DENSE:
        if R_k is None or R_v is None:
            raise ValueError("dense rotation needs R_k and R_v")
        _need_shape(R_k, torch.float32, "R_k", (Hkv, D, D))
        _need_shape(R_v, torch.float32, "R_v", (Hkv, D, D))
        _need(R_k, torch.float32, "R_k", (Hkv, D, D))
        _need(R_v, torch.float32, "R_v", (Hkv, D, D))
    elif mode == KVQ_ROT_PERM_FWHT:
        if perm is None:
            raise ValueError("permutation + FWHT rotation needs perm")
        _need(perm, torch.int32, "perm", (2, Hkv, D))
    else:
        raise ValueError("unknown rotation mode %r" % (mode,))


def _sink_arrays(cache, B, Hkv, sink_fp16, identified_sinks, device):
    """fp16 sink rows, and for identified sinks the position list and counts."""
    if identified_sinks and sink_fp16 < 1:
        raise ValueError("identified sinks need sink_fp16 >= 1")
    if sink_fp16 > 0:
        cache.k_sink = torch.zeros((B, Hkv, sink_fp16, D), dtype=torch.float16, device=device)
        cache.v_sink = torch.zeros_like(cache.k_sink)
    else:
        cache.k_sink = cache.v_sink = None
    if identified_sinks:
        cache.sink_pos = torch.zeros((B, sink_fp16), dtype=torch.int32, device=device)
        cache.sink_count = torch.zeros(B, dtype=torch.int32, device=device)
    else:
        cache.sink_pos = cache.sink_count = None


def _desc(cache, table=0, num_blocks=0):
    p = lambda t: 0 if t is None else t.data_ptr()
    return CacheDesc(cache.B, cache.Hkv, D, GROUP, cache.capacity, cache.sink_fp16,
                     cache.blocks.data_ptr(), p(cache.k_sink), p(cache.v_sink),
                     cache.status.data_ptr(), table, num_blocks, p(cache.sink_pos),
                     p(cache.sink_count))


class KVCache:
    """A packed INT2 cache for B sequences x Hkv heads (memory owned by torch).
    sink_fp16 rows of fp16 sinks per (sequence, head): the leading positions,
    or with identified_sinks=True the positions kvq_identify_sinks picks
    (listed in sink_pos [B][sink_fp16], sink_count [B])."""

    def __init__(self, B, Hkv, capacity, sink_fp16=0, device="cuda", identified_sinks=False):
        nbytes = lib().kvq_cache_bytes(B, Hkv, capacity)
        if nbytes == 0:
            raise ValueError("bad cache shape B=%d Hkv=%d capacity=%d" % (B, Hkv, capacity))
        self.B, self.Hkv, self.capacity, self.sink_fp16 = B, Hkv, capacity, sink_fp16
        self.blocks = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        _sink_arrays(self, B, Hkv, sink_fp16, identified_sinks, device)
        self.status = torch.zeros(2, dtype=torch.int32, device=device)   # errors, append counter
        self.desc = _desc(self)

    def block_view(self):
        """blocks as uint8 [B][Hkv][capacity/16][1536]."""
        return self.blocks.view(self.B, self.Hkv, self.capacity // BLOCK_TOKENS, BLOCK_BYTES)


class PagedKVCache(KVCache):
    """A paged cache: a pool of num_blocks blocks (each 16 tokens x Hkv heads x
    1536 bytes) and an int32 block table [B][capacity/16] mapping every
    sequence's logical blocks to pool blocks (memory owned by torch)."""

    def __init__(self, B, Hkv, capacity, num_blocks, block_table, sink_fp16=0, device="cuda",
                 identified_sinks=False):
        if capacity % BLOCK_TOKENS or num_blocks < 1:
            raise ValueError("bad paged cache shape")
        _need(block_table, torch.int32, "block_table", (B, capacity // BLOCK_TOKENS))
        self.B, self.Hkv, self.capacity, self.sink_fp16 = B, Hkv, capacity, sink_fp16
        self.num_blocks, self.block_table = num_blocks, block_table
        self.blocks = torch.zeros(num_blocks * Hkv * BLOCK_BYTES, dtype=torch.uint8, device=device)
        _sink_arrays(self, B, Hkv, sink_fp16, identified_sinks, device)
        self.status = torch.zeros(2, dtype=torch.int32, device=device)
        self.desc = _desc(self, block_table.data_ptr(), num_blocks)

    def block_view(self):
        """The pool as uint8 [num_blocks][Hkv][1536]."""
        return self.blocks.view(self.num_blocks, self.Hkv, BLOCK_BYTES)

    def logical_view(self):
        """The blocks gathered into the contiguous layout [B][Hkv][capacity/16][1536]
        (a copy; entries outside the pool must not occur)."""
        t = self.block_table.long()
        return self.block_view()[t].permute(0, 2, 1, 3).contiguous()


def kvq_cache_bytes(B, Hkv, capacity):
    return lib().kvq_cache_bytes(B, Hkv, capacity)


def kvq_rotate_quantize_append(K, V, mode, R_k, R_v, perm, cache, seq_lens, stream=None):
    """K, V fp16 [B][T][Hkv][128]; seq_lens int32 [B] (updated in place)."""
    _need_rotation(mode, R_k, R_v, perm, cache.Hkv)
    B, T, Hkv, d = K.shape
    _need(K, torch.float16, "K", (cache.B, T, cache.Hkv, D))
    _need(V, torch.float16, "V", K.shape)
    _need(seq_lens, torch.int32, "seq_lens", (cache.B,))
    _check("kvq_rotate_quantize_append",
           lib().kvq_rotate_quantize_append(_ptr(K), _ptr(V), T, mode, _ptr(R_k), _ptr(R_v),
                                            _ptr(perm), C.byref(cache.desc), _ptr(seq_lens),
                                            _stream(stream, K)))


def kvq_identify_sinks(act, tau, cache, seq_lens, stream=None):
    """act fp32 [B][T]: activation magnitudes of the next T tokens (call just
    before appending them); seq_lens int32 [B], the lengths before that
    append.  Tokens with act >= tau take the free fp16 sink rows."""
    _need(act, torch.float32, "act")
    _need(seq_lens, torch.int32, "seq_lens", (cache.B,))
    if act.dim() != 2 or act.shape[0] != cache.B:
        raise ValueError("act must have shape (B, T)")
    _check("kvq_identify_sinks",
           lib().kvq_identify_sinks(_ptr(act), act.shape[1], float(tau), C.byref(cache.desc),
                                    _ptr(seq_lens), _stream(stream, act)))


def _sm_count(device=None):
    """SM count of `device` (default: the current CUDA device); the library
    sizes its split from the SM count of the device the call runs on."""
    d = torch.device("cuda" if device is None else device)
    idx = d.index if d.index is not None else torch.cuda.current_device()
    return torch.cuda.get_device_properties(idx).multi_processor_count


def kvq_decode_workspace_size(B, Hq, Hkv, max_ctx, sm_count=None):
    if sm_count is None:
        sm_count = _sm_count()
    return lib().kvq_decode_workspace_size(B, Hq, Hkv, max_ctx, sm_count)


def decode_workspace(B, Hq, Hkv, max_ctx, device="cuda"):
    n = kvq_decode_workspace_size(B, Hq, Hkv, max_ctx, _sm_count(device))
    if n == 0:
        raise ValueError("bad decode shape")
    return torch.empty(n, dtype=torch.uint8, device=device)


def kvq_decode_attention(Q, cache, mode, R_k, R_v, perm, seq_lens, sink_fp16, max_ctx,
                         workspace, out, stream=None):
    """Q fp16 [B][Hq][128] -> out fp16 [B][Hq][128]; seq_lens int32 [B] on device."""
    _need_rotation(mode, R_k, R_v, perm, cache.Hkv)
    B, Hq, d = Q.shape
    _need(Q, torch.float16, "Q", (cache.B, Hq, D))
    _need(out, torch.float16, "out", Q.shape)
    _need(seq_lens, torch.int32, "seq_lens", (cache.B,))
    _need(workspace, torch.uint8, "workspace")
    _check("kvq_decode_attention",
           lib().kvq_decode_attention(_ptr(Q), Hq, C.byref(cache.desc), mode, _ptr(R_k), _ptr(R_v),
                                      _ptr(perm), _ptr(seq_lens), sink_fp16, max_ctx,
                                      _ptr(workspace), workspace.numel(), _ptr(out),
                                      _stream(stream, Q)))


def kvq_append_decode(K, V, Q, cache, mode, R_k, R_v, perm, seq_lens, max_ctx, workspace, out,
                      stream=None):
    """One serving step: append K, V fp16 [B][T][Hkv][128] (seq_lens int32 [B]
    advance by T on the device), then decode Q fp16 [B][Hq][128] into out over
    the updated cache."""
    _need_rotation(mode, R_k, R_v, perm, cache.Hkv)
    B, T, Hkv, d = K.shape
    _need(K, torch.float16, "K", (cache.B, T, cache.Hkv, D))
    _need(V, torch.float16, "V", K.shape)
    _need(Q, torch.float16, "Q")
    _need(out, torch.float16, "out", Q.shape)
    _need(seq_lens, torch.int32, "seq_lens", (cache.B,))
    _need(workspace, torch.uint8, "workspace")
    if Q.dim() != 3 or Q.shape[0] != cache.B or Q.shape[2] != D:
        raise ValueError("Q must have shape (B, Hq, 128)")
    _check("kvq_append_decode",
           lib().kvq_append_decode(_ptr(K), _ptr(V), T, _ptr(Q), Q.shape[1], C.byref(cache.desc),
                                   mode, _ptr(R_k), _ptr(R_v), _ptr(perm), _ptr(seq_lens),
                                   max_ctx, _ptr(workspace), workspace.numel(), _ptr(out),
                                   _stream(stream, Q)))


def _need_host(t, dtype, name, shape=None):
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if t.is_cuda or not t.is_contiguous():
        raise ValueError("%s must be a contiguous host tensor (pinned for overlap)" % name)
    if shape is not None and t.shape != shape:
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))


def kvq_step_workspace_size(B, T, Hq, Hkv, max_ctx, sm_count=None):
    if sm_count is None:
        sm_count = _sm_count()
    return lib().kvq_step_workspace_size(B, T, Hq, Hkv, max_ctx, sm_count)


def step_workspace(B, T, Hq, Hkv, max_ctx, device="cuda"):
    n = kvq_step_workspace_size(B, T, Hq, Hkv, max_ctx, _sm_count(device))
    if n == 0:
        raise ValueError("bad step shape")
    return torch.empty(n, dtype=torch.uint8, device=device)


def kvq_append_decode_host(K_host, V_host, Q_host, cache, mode, R_k, R_v, perm, seq_lens, max_ctx,
                           workspace, out_host, stream=None):
    """The serving step with host tensors (pin them): K, V fp16 [B][T][Hkv][128]
    and Q fp16 [B][Hq][128] are copied in, appended and decoded, and the output
    copied back into out_host, all queued on the stream (synchronise before
    reading out_host).  K, V and Q that are consecutive views of one buffer
    (V right after K, Q right after V) go in with a single copy.
    workspace: step_workspace(...) on the device."""
    _need_rotation(mode, R_k, R_v, perm, cache.Hkv)
    B, T, Hkv, d = K_host.shape
    _need_host(K_host, torch.float16, "K_host", (cache.B, T, cache.Hkv, D))
    _need_host(V_host, torch.float16, "V_host", K_host.shape)
    _need_host(Q_host, torch.float16, "Q_host")
    _need_host(out_host, torch.float16, "out_host", Q_host.shape)
    _need(seq_lens, torch.int32, "seq_lens", (cache.B,))
    _need(workspace, torch.uint8, "workspace")
    if Q_host.dim() != 3 or Q_host.shape[0] != cache.B or Q_host.shape[2] != D:
        raise ValueError("Q_host must have shape (B, Hq, 128)")
    _check("kvq_append_decode_host",
           lib().kvq_append_decode_host(_ptr(K_host), _ptr(V_host), T, _ptr(Q_host),
                                        Q_host.shape[1], C.byref(cache.desc), mode, _ptr(R_k),
                                        _ptr(R_v), _ptr(perm), _ptr(seq_lens), max_ctx,
                                        _ptr(workspace), workspace.numel(), _ptr(out_host),
                                        _stream(stream, workspace)))


class HostStep:
    """kvq_append_decode_host prepared once: every argument is checked here,
    and run() queues the step (copies in, append, decode, copy out) with one
    C call and no per-call Python checks, for a serving loop whose buffers
    stay the same from step to step (their contents change: new K/V rows,
    new queries).  The tensors must stay alive and keep their shapes; the
    stream is the one given (or current) at construction.  run() may name
    another int32 [B] device tensor of lengths for that step."""

    def __init__(self, K_host, V_host, Q_host, cache, mode, R_k, R_v, perm, seq_lens, max_ctx,
                 workspace, out_host, stream=None):
        _need_rotation(mode, R_k, R_v, perm, cache.Hkv)
        B, T, Hkv, d = K_host.shape
        _need_host(K_host, torch.float16, "K_host", (cache.B, T, cache.Hkv, D))
        _need_host(V_host, torch.float16, "V_host", K_host.shape)
        _need_host(Q_host, torch.float16, "Q_host")
        _need_host(out_host, torch.float16, "out_host", Q_host.shape)
        _need(seq_lens, torch.int32, "seq_lens", (cache.B,))
        _need(workspace, torch.uint8, "workspace")
        if Q_host.dim() != 3 or Q_host.shape[0] != cache.B or Q_host.shape[2] != D:
            raise ValueError("Q_host must have shape (B, Hq, 128)")
        self._keep = (K_host, V_host, Q_host, cache, R_k, R_v, perm, seq_lens, workspace,
                      out_host)
        self._fn = lib().kvq_append_decode_host
        self._sl_shape = seq_lens.shape
        self._sl_dev = seq_lens.device
        self._args = [_ptr(K_host), _ptr(V_host), T, _ptr(Q_host), Q_host.shape[1],
                      C.byref(cache.desc), mode, _ptr(R_k), _ptr(R_v), _ptr(perm),
                      _ptr(seq_lens), max_ctx, _ptr(workspace), workspace.numel(),
                      _ptr(out_host), _stream(stream, workspace)]

    def run(self, seq_lens=None):
        args = self._args
        if seq_lens is not None:
            if (seq_lens.dtype is not torch.int32 or seq_lens.shape != self._sl_shape or
                    seq_lens.device != self._sl_dev or not seq_lens.is_contiguous()):
                raise ValueError("seq_lens must be a contiguous int32 tensor like the plan's")
            args = list(args)
            args[10] = seq_lens.data_ptr()
        code = self._fn(*args)
        if code:
            raise KvqError("kvq_append_decode_host", code)


KVQ_DECODE_OUT_ROTATED = 1


def kvq_decode_attention_ex(Q, cache, mode, R_k, R_v, perm, seq_lens, sink_fp16, max_ctx,
                            workspace, out, flags=0, stream=None):
    """Q fp16 [B][Hq][q_len][128] -> out fp16 [B][Hq][q_len][128]: q_len new tokens
    per sequence, each attending causally; flags: KVQ_DECODE_OUT_ROTATED."""
    _need_rotation(mode, R_k, R_v, perm, cache.Hkv)
    B, Hq, q_len, d = Q.shape
    _need(Q, torch.float16, "Q", (cache.B, Hq, q_len, D))
    _need(out, torch.float16, "out", Q.shape)
    _need(seq_lens, torch.int32, "seq_lens", (cache.B,))
    _need(workspace, torch.uint8, "workspace")
    _check("kvq_decode_attention_ex",
           lib().kvq_decode_attention_ex(_ptr(Q), Hq, q_len, flags, C.byref(cache.desc), mode,
                                         _ptr(R_k), _ptr(R_v), _ptr(perm), _ptr(seq_lens),
                                         sink_fp16, max_ctx, _ptr(workspace), workspace.numel(),
                                         _ptr(out), _stream(stream, Q)))


def kvq_decode_attention_adapter(Q, cache, mode, R_k, R_v, perm, U_k, V_k, seq_lens, sink_fp16,
                                 max_ctx, workspace, out, flags=0, stream=None):
    """Decode with KVLinC key correction adapters U_k, V_k fp32 [Hkv][128][r]:
    every INT2 key k^ (model basis) is scored as k^ + (k^ . U) . V^T.
    Q fp16 [B][Hq][128] or [B][Hq][q_len][128] -> out of the same shape."""
    _need_rotation(mode, R_k, R_v, perm, cache.Hkv)
    if U_k is None or V_k is None or U_k.dim() != 3:
        raise ValueError("U_k and V_k must be [Hkv][128][rank] tensors")
    _need(U_k, torch.float32, "U_k", (cache.Hkv, D, U_k.shape[2]))
    _need(V_k, torch.float32, "V_k", U_k.shape)
    if Q.dim() == 3:
        B, Hq, d = Q.shape
        q_len = 1
    else:
        B, Hq, q_len, d = Q.shape
    _need(Q, torch.float16, "Q", (cache.B, Hq, D) if Q.dim() == 3 else (cache.B, Hq, q_len, D))
    _need(out, torch.float16, "out", Q.shape)
    _need(seq_lens, torch.int32, "seq_lens", (cache.B,))
    _need(workspace, torch.uint8, "workspace")
    _check("kvq_decode_attention_adapter",
           lib().kvq_decode_attention_adapter(_ptr(Q), Hq, q_len, flags, C.byref(cache.desc), mode,
                                              _ptr(R_k), _ptr(R_v), _ptr(perm), _ptr(U_k),
                                              _ptr(V_k), U_k.shape[2], _ptr(seq_lens), sink_fp16,
                                              max_ctx, _ptr(workspace), workspace.numel(),
                                              _ptr(out), _stream(stream, Q)))


def kvq_decode_attention_timed(Q, cache, mode, R_k, R_v, perm, seq_lens, sink_fp16, max_ctx,
                               workspace, out, ev_begin, ev_end, stream=None):
    """kvq_decode_attention that also records torch.cuda.Events ev_begin /
    ev_end (already recorded once, so they exist) around the kernel that
    streams the packed cache."""
    _need_rotation(mode, R_k, R_v, perm, cache.Hkv)
    B, Hq, d = Q.shape
    _need(Q, torch.float16, "Q", (cache.B, Hq, D))
    _need(out, torch.float16, "out", Q.shape)
    _need(seq_lens, torch.int32, "seq_lens", (cache.B,))
    _need(workspace, torch.uint8, "workspace")
    _check("kvq_decode_attention_timed",
           lib().kvq_decode_attention_timed(_ptr(Q), Hq, C.byref(cache.desc), mode, _ptr(R_k),
                                            _ptr(R_v), _ptr(perm), _ptr(seq_lens), sink_fp16,
                                            max_ctx, _ptr(workspace), workspace.numel(), _ptr(out),
                                            _stream(stream, Q), C.c_void_p(ev_begin.cuda_event),
                                            C.c_void_p(ev_end.cuda_event)))


def kvq_decode_attention_noalloc(Q, cache, mode, R_k, R_v, perm, seq_lens, sink_fp16, max_ctx,
                                 out, stream=None):
    """kvq_decode_attention for callers that cannot allocate device memory:
    no workspace argument, the library's fixed device array serves instead
    (see include/kvq.h for its size and the sharing rules)."""
    _need_rotation(mode, R_k, R_v, perm, cache.Hkv)
    B, Hq, d = Q.shape
    _need(Q, torch.float16, "Q", (cache.B, Hq, D))
    _need(out, torch.float16, "out", Q.shape)
    _need(seq_lens, torch.int32, "seq_lens", (cache.B,))
    _check("kvq_decode_attention_noalloc",
           lib().kvq_decode_attention_noalloc(_ptr(Q), Hq, C.byref(cache.desc), mode, _ptr(R_k),
                                              _ptr(R_v), _ptr(perm), _ptr(seq_lens), sink_fp16,
                                              max_ctx, _ptr(out), _stream(stream, Q)))


def kvq_get_status(cache, stream=None):
    v = C.c_int32(0)
    _check("kvq_get_status", lib().kvq_get_status(C.byref(cache.desc), _stream(stream, cache.status),
                                                  C.byref(v)))
    return v.value


def kvq_clear_status(cache, stream=None):
    _check("kvq_clear_status", lib().kvq_clear_status(C.byref(cache.desc),
                                                      _stream(stream, cache.status)))


def kvq_debug_rotate_f32(X, mode, R=None, perm=None, variant=0, stream=None):
    """X fp16 [N][128] -> fp32 [N][128] rotated by one head's rotation."""
    _need(X, torch.float16, "X")
    N = X.shape[0]
    out = torch.empty((N, D), dtype=torch.float32, device=X.device)
    _check("kvq_debug_rotate_f32",
           lib().kvq_debug_rotate_f32(_ptr(X), N, mode, _ptr(R), _ptr(perm), variant, _ptr(out),
                                      _stream(stream, X)))
    return out


def kvq_debug_quantize_f32(Xrot, stream=None):
    """fp32 [N][128] -> (codes uint8 [N][32] logical packing, meta int16 [N][4][2] {s, z})."""
    _need(Xrot, torch.float32, "Xrot")
    N = Xrot.shape[0]
    codes = torch.empty((N, 32), dtype=torch.uint8, device=Xrot.device)
    meta = torch.empty((N, 4, 2), dtype=torch.int16, device=Xrot.device)
    _check("kvq_debug_quantize_f32",
           lib().kvq_debug_quantize_f32(_ptr(Xrot), N, _ptr(codes), _ptr(meta),
                                        _stream(stream, Xrot)))
    return codes, meta


# --- pre-RoPE grouped-head key rotation ---------------------------------------------------

def kvq_prerope_append(K, V, group_heads, perm, cache, seq_lens, stream=None):
    """K (pre-RoPE), V fp16 [B][T][Hkv][128]; perm int32 [2][Hkv*128] (plane 0:
    Hkv/group_heads key permutations of 128*group_heads entries; plane 1: one
    value permutation of 128 per head); seq_lens int32 [B], updated."""
    B, T, Hkv, d = K.shape
    _need(K, torch.float16, "K", (cache.B, T, cache.Hkv, D))
    _need(V, torch.float16, "V", K.shape)
    _need(seq_lens, torch.int32, "seq_lens", (cache.B,))
    _need(perm, torch.int32, "perm", (2, cache.Hkv * D))
    _check("kvq_prerope_append",
           lib().kvq_prerope_append(_ptr(K), _ptr(V), T, group_heads, _ptr(perm),
                                    C.byref(cache.desc), _ptr(seq_lens), _stream(stream, K)))


def kvq_prerope_workspace_size(B, Hq, Hkv, group_heads, max_ctx, sm_count=None):
    if sm_count is None:
        sm_count = _sm_count()
    return lib().kvq_prerope_workspace_size(B, Hq, Hkv, group_heads, max_ctx, sm_count)


def prerope_workspace(B, Hq, Hkv, group_heads, max_ctx, device="cuda"):
    n = kvq_prerope_workspace_size(B, Hq, Hkv, group_heads, max_ctx, _sm_count(device))
    if n == 0:
        raise ValueError("bad pre-RoPE decode shape")
    return torch.empty(n, dtype=torch.uint8, device=device)


def kvq_prerope_decode(Q, cache, group_heads, perm, rope_base, seq_lens, max_ctx, workspace, out,
                       stream=None):
    """Q fp16 [B][Hq][128] post-RoPE queries -> out fp16 [B][Hq][128]."""
    B, Hq, d = Q.shape
    _need(Q, torch.float16, "Q", (cache.B, Hq, D))
    _need(out, torch.float16, "out", Q.shape)
    _need(seq_lens, torch.int32, "seq_lens", (cache.B,))
    _need(workspace, torch.uint8, "workspace")
    _need(perm, torch.int32, "perm", (2, cache.Hkv * D))
    _check("kvq_prerope_decode",
           lib().kvq_prerope_decode(_ptr(Q), Hq, C.byref(cache.desc), group_heads, _ptr(perm),
                                    float(rope_base), _ptr(seq_lens), max_ctx, _ptr(workspace),
                                    workspace.numel(), _ptr(out), _stream(stream, Q)))


def kvq_debug_rotate_group_f32(X, group_heads, perm, stream=None):
    """X fp16 [N][128*group_heads] -> fp32 rows rotated by one group permutation + FWHT."""
    _need(X, torch.float16, "X")
    _need(perm, torch.int32, "perm", (D * group_heads,))
    N = X.shape[0]
    out = torch.empty((N, D * group_heads), dtype=torch.float32, device=X.device)
    _check("kvq_debug_rotate_group_f32",
           lib().kvq_debug_rotate_group_f32(_ptr(X), N, group_heads, _ptr(perm), _ptr(out),
                                            _stream(stream, X)))
    return out


def kvq_debug_wait_timeout(src, poll_limit, status, stream=None):
    """Runs the bounded-wait failure path once: src uint8 [1536] on the device,
    status int32 device word(s) (KVQ_DEV_TIMEOUT is ORed into status[0]).
    Returns int32 [3] on the device: gave up (1), stages lost by the drain,
    byte sum of the copy as it landed in shared memory."""
    _need(src, torch.uint8, "src", (BLOCK_BYTES,))
    _need(status, torch.int32, "status")
    result = torch.full((3,), -1, dtype=torch.int32, device=src.device)
    _check("kvq_debug_wait_timeout",
           lib().kvq_debug_wait_timeout(_ptr(src), int(poll_limit), _ptr(status), _ptr(result),
                                        _stream(stream, src)))
    return result
