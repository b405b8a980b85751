"""Python binding of libkvpop.so (the KVpop fixed-budget KV cache C ABI).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels behind include/kvpop.h.  PyTorch supplies device memory and streams.
Importing this module loads the in-tree libkvpop.so and fails loudly if it is
missing; there is no fallback implementation.

Names follow the C ABI: kvpop_cache_bytes, kvpop_create, kvpop_prefill,
kvpop_decode_step, kvpop_inspect, kvpop_get_layout, kvpop_get_error,
kvpop_clear_error, kvpop_debug_poison_error, kvpop_destroy,
kvpop_status_string.  `KVPopCache` bundles a handle with its device buffer.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
# KVPOP_LIBRARY may point at another build of the same library (e.g. a tuning variant).
LIB_PATH = os.environ.get("KVPOP_LIBRARY") or os.path.join(_HERE, "libkvpop.so")

KVPOP_OK = 0
KVPOP_ERR_INVALID_ARG = -1
KVPOP_ERR_BAD_SHAPE = -2
KVPOP_ERR_ORDER = -3
KVPOP_ERR_CONTEXT_OVERFLOW = -4
KVPOP_ERR_CUDA = -5
KVPOP_ERR_DEVICE = -6
KVPOP_ERR_TIMEOUT = -7
KVPOP_ERR_SCRATCH_LIMIT = -8

KVPOP_NOALLOC_SCRATCH_BYTES = 16 << 20   # static split-K buffer behind decode_step_noalloc

KVPOP_DTYPE_F32 = 0
KVPOP_DTYPE_BF16 = 1
KVPOP_FLAG_EXTERNAL_SCORES = 1
KVPOP_FLAG_DEBUG_CHECKS = 2

KVPOP_DEVERR_CONTEXT_OVERFLOW = 1
KVPOP_DEVERR_TIMEOUT = 2
KVPOP_DEVERR_BAD_INDEX = 4
KVPOP_DEVERR_NAN_SCORE = 8
KVPOP_DEVERR_STATE_MISMATCH = 16

EXPORTED_SYMBOLS = (
    "kvpop_cache_bytes", "kvpop_create", "kvpop_prefill", "kvpop_decode_step", "kvpop_decode_append",
    "kvpop_decode_attend", "kvpop_inspect",
    "kvpop_get_layout", "kvpop_get_error", "kvpop_clear_error", "kvpop_debug_poison_error",
    "kvpop_destroy", "kvpop_status_string", "kvpop_decode_step_noalloc",
    "kvpop_prefill_attention_workspace_bytes", "kvpop_prefill_attention", "kvpop_prefill_with_attention",
    "kvpop_debug_set_hook", "kvpop_prefill_attention_from_cutoffs",
)


class kvpop_config(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("n_layers", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("sinks", ctypes.c_int32),
        ("window", ctypes.c_int32), ("topk", ctypes.c_int32), ("delay", ctypes.c_int32),
        ("ref_context", ctypes.c_int32), ("compression_ratio", ctypes.c_float),
        ("max_context", ctypes.c_int32), ("max_prefill_chunk", ctypes.c_int32),
        ("dtype", ctypes.c_int32), ("scorer_hidden", ctypes.c_int32),
        ("w1", ctypes.c_void_p), ("b1", ctypes.c_void_p), ("w2", ctypes.c_void_p), ("b2", ctypes.c_void_p),
        ("flags", ctypes.c_uint32), ("log_decay", ctypes.c_void_p),
        ("scorer_kind", ctypes.c_int32), ("mlstm_p", ctypes.c_int32), ("mlstm_dv", ctypes.c_int32),
        ("mlstm_w", ctypes.c_void_p),
    ]


KVPOP_SCORER_MLP = 0
KVPOP_SCORER_MLSTM = 1


def mlstm_head_floats(p: int, dv: int, d: int) -> int:
    """Floats of one (layer, KV head) block of the mLSTM weights (include/kvpop.h
    KVPOP_MLSTM_HEAD_FLOATS): W_q, W_k [p][2d], W_v [dv][2d], w_i, w_f [2d],
    then w_o [dv], b_i, b_f, b_o, padded to a multiple of 4."""
    return (2 * p + dv + 2) * 2 * d + ((dv + 3 + 3) // 4) * 4


class kvpop_layout_info(ctypes.Structure):
    _fields_ = [
        ("kv_offset", ctypes.c_size_t), ("kv_layer_stride", ctypes.c_size_t),
        ("pos_offset", ctypes.c_size_t), ("pos_layer_stride", ctypes.c_size_t),
        ("score_offset", ctypes.c_size_t), ("score_layer_stride", ctypes.c_size_t),
        ("state_offset", ctypes.c_size_t), ("state_layer_stride", ctypes.c_size_t),
        ("slots_per_unit", ctypes.c_int32), ("units", ctypes.c_int32), ("row_bytes", ctypes.c_int32),
        ("topk_base", ctypes.c_int32),
    ]


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"libkvpop.so not built at {path}: run "
                          "`python fixed_budget_kv_kvpop_b200/csrc/build.py` (no CPU fallback exists)")
    lib = ctypes.CDLL(path)
    P, I32, U32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint32, ctypes.c_size_t
    sig = {
        "kvpop_cache_bytes": ([ctypes.POINTER(kvpop_config), ctypes.POINTER(SZ)], ctypes.c_int),
        "kvpop_create": ([ctypes.POINTER(kvpop_config), P, SZ, ctypes.POINTER(P)], ctypes.c_int),
        "kvpop_prefill": ([P, I32, P, P, I32, P, P], ctypes.c_int),
        "kvpop_decode_step": ([P, I32, P, P, P, P, P, P], ctypes.c_int),
        "kvpop_decode_append": ([P, I32, P, P, P, P], ctypes.c_int),
        "kvpop_decode_attend": ([P, I32, P, P, P], ctypes.c_int),
        "kvpop_inspect": ([P, I32, P, P, P, P], ctypes.c_int),
        "kvpop_get_layout": ([P, ctypes.POINTER(kvpop_layout_info)], ctypes.c_int),
        "kvpop_get_error": ([P, ctypes.POINTER(I32)], ctypes.c_int),
        "kvpop_clear_error": ([P, P], ctypes.c_int),
        "kvpop_debug_poison_error": ([P, I32, P], ctypes.c_int),
        "kvpop_destroy": ([P], ctypes.c_int),
        "kvpop_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "kvpop_decode_step_noalloc": ([P, I32, P, P, P, P, P, P], ctypes.c_int),
        "kvpop_prefill_attention_workspace_bytes": ([P, I32, ctypes.POINTER(SZ)], ctypes.c_int),
        "kvpop_prefill_attention": ([P, I32, P, P, P, I32, P, P, P, P, SZ, P], ctypes.c_int),
        "kvpop_prefill_with_attention": ([P, I32, P, P, P, I32, P, P, P, P, SZ, P], ctypes.c_int),
        "kvpop_debug_set_hook": ([P, I32], ctypes.c_int),
        "kvpop_prefill_attention_from_cutoffs": ([P, I32, P, P, P, I32, P, P, P, SZ, P], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


lib = load_library()


class KVPopError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib.kvpop_status_string(status).decode()} ({status})")


def _check(status: int, what: str) -> None:
    if status != KVPOP_OK:
        raise KVPopError(status, what)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return stream.cuda_stream or None


_DTYPE_NAMES = {"f32": KVPOP_DTYPE_F32, "float32": KVPOP_DTYPE_F32, "fp32": KVPOP_DTYPE_F32,
                "bf16": KVPOP_DTYPE_BF16, "bfloat16": KVPOP_DTYPE_BF16}


def dtype_code(dtype) -> int:
    """KVPOP_DTYPE_* of an element-type name ('f32', 'float32', 'fp32',
    'bf16', 'bfloat16') or of torch.float32 / torch.bfloat16; anything else
    raises ValueError."""
    if isinstance(dtype, str):
        if dtype in _DTYPE_NAMES:
            return _DTYPE_NAMES[dtype]
    else:
        import torch
        if dtype == torch.float32:
            return KVPOP_DTYPE_F32
        if dtype == torch.bfloat16:
            return KVPOP_DTYPE_BF16
    raise ValueError(f"unsupported element type {dtype!r}: use one of {sorted(_DTYPE_NAMES)}")


def _torch_dtype(code: int):
    import torch
    return torch.float32 if code == KVPOP_DTYPE_F32 else torch.bfloat16


def check_tensor(t, name: str, shape, dtype, device) -> None:
    """Raises ValueError unless `t` is a contiguous CUDA tensor on `device`
    (a torch.device) with exactly `shape` and `dtype`.  The C ABI sees only
    raw pointers, so every tensor is checked here before its address is
    passed on."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.device.type != "cuda" or t.device != device:
        raise ValueError(f"{name}: on {t.device}, the cache lives on {device}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


def make_config(*, batch, n_layers, n_q_heads, n_kv_heads, head_dim, sinks, window, topk, delay=0,
                ref_context=0, compression_ratio=0.0, max_context=None, max_prefill_chunk=0,
                dtype="bf16", scorer_hidden=64, w1=None, b1=None, w2=None, b2=None,
                external_scores=False, debug_checks=False, log_decay=None, scorer="mlp", mlstm_p=0,
                mlstm_dv=0, mlstm_w=None) -> kvpop_config:
    """log_decay: optional device fp32 tensor [n_layers][n_kv_heads] of
    ln(gamma_h) <= 0 (temporal decay); max_context defaults to 2^30, or 2^24
    with decay.  scorer: 'mlp' (w1/b1/w2/b2; the linear scorer when
    scorer_hidden = 0) or 'mlstm' (mlstm_p, mlstm_dv and the packed device
    weights mlstm_w [n_layers][n_kv_heads][mlstm_head_floats(p, dv, d)])."""
    if scorer not in ("mlp", "mlstm"):
        raise ValueError(f"unknown scorer {scorer!r}: 'mlp' or 'mlstm'")
    if max_context is None:
        max_context = (1 << 24) if log_decay is not None else (1 << 30)
    c = kvpop_config()
    c.batch, c.n_layers, c.n_q_heads, c.n_kv_heads, c.head_dim = batch, n_layers, n_q_heads, n_kv_heads, head_dim
    c.sinks, c.window, c.topk, c.delay = sinks, window, topk, delay
    c.ref_context, c.compression_ratio = ref_context, compression_ratio
    c.max_context, c.max_prefill_chunk = max_context, max_prefill_chunk
    c.dtype = dtype_code(dtype)
    c.scorer_hidden = scorer_hidden
    c.w1, c.b1, c.w2, c.b2 = _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2)
    c.flags = (KVPOP_FLAG_EXTERNAL_SCORES if external_scores else 0) | (KVPOP_FLAG_DEBUG_CHECKS if debug_checks else 0)
    c.log_decay = _ptr(log_decay)
    c.scorer_kind = KVPOP_SCORER_MLSTM if scorer == "mlstm" else KVPOP_SCORER_MLP
    c.mlstm_p, c.mlstm_dv = mlstm_p, mlstm_dv
    c.mlstm_w = _ptr(mlstm_w)
    return c


def cache_bytes(cfg: kvpop_config, library=None) -> int:
    n = ctypes.c_size_t(0)
    _check((library or lib).kvpop_cache_bytes(ctypes.byref(cfg), ctypes.byref(n)), "kvpop_cache_bytes")
    return n.value


class KVPopCache:
    """A handle plus the device buffer it lives in (allocated with torch).

    The scorer weights passed to make_config must stay alive as long as this
    object; they are kept referenced here.
    """

    def __init__(self, cfg: kvpop_config, device=None, keepalive=(), library=None):
        """library: another build of the same library loaded with
        load_library (the test-hook build, for instance); default libkvpop.so."""
        import torch
        self.cfg = cfg
        self._lib = library or lib
        self._keep = tuple(keepalive)
        self.nbytes = cache_bytes(cfg, self._lib)
        self.buffer = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device or "cuda")
        base = self.buffer.data_ptr()
        self._off = (-base) % 256
        self.handle = ctypes.c_void_p()
        _check(self._lib.kvpop_create(ctypes.byref(cfg), ctypes.c_void_p(base + self._off), self.nbytes,
                                ctypes.byref(self.handle)), "kvpop_create")
        self.device = self.buffer.device
        self.dtype = _torch_dtype(cfg.dtype)

    # -- argument checks (shapes from include/kvpop.h) --
    def _elems(self, name, t, shape):
        check_tensor(t, name, shape, self.dtype, self.device)

    def _f32(self, name, t, shape):
        import torch
        check_tensor(t, name, shape, torch.float32, self.device)

    def _dims(self):
        c = self.cfg
        return c.batch, c.n_q_heads, c.n_kv_heads, c.head_dim

    def __del__(self):
        h = getattr(self, "handle", None)
        if h:
            self._lib.kvpop_destroy(h)
            self.handle = None

    def prefill(self, layer: int, k, v, ext_scores=None, stream=None):
        n = int(k.shape[2]) if k is not None else 0
        if k is not None or v is not None:
            b, _, hkv, d = self._dims()
            self._elems("k", k, (b, hkv, n, d))
            self._elems("v", v, (b, hkv, n, d))
            if ext_scores is not None:
                self._f32("ext_scores", ext_scores, (b, hkv, n))
        _check(self._lib.kvpop_prefill(self.handle, layer, _ptr(k), _ptr(v), n, _ptr(ext_scores),
                                 _stream_ptr(stream)), "kvpop_prefill")

    def _check_step(self, q, k_new, v_new, out, ext_score):
        b, hq, hkv, d = self._dims()
        self._elems("q", q, (b, hq, d))
        self._elems("k_new", k_new, (b, hkv, d))
        self._elems("v_new", v_new, (b, hkv, d))
        self._elems("out", out, (b, hq, d))
        if ext_score is not None:
            self._f32("ext_score", ext_score, (b, hkv))

    def decode_step(self, layer: int, q, k_new, v_new, out, ext_score=None, stream=None):
        self._check_step(q, k_new, v_new, out, ext_score)
        _check(self._lib.kvpop_decode_step(self.handle, layer, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(out),
                                     _ptr(ext_score), _stream_ptr(stream)), "kvpop_decode_step")

    def decode_step_noalloc(self, layer: int, q, k_new, v_new, out, ext_score=None, stream=None):
        """decode_step for callers that cannot allocate device memory: the
        split-K scratch comes from the library's static 16 MiB buffer instead
        of this handle's buffer, so the call allocates nothing.  Its first
        call on a device looks up that buffer once (make it before any stream
        capture); calls that overlap on the GPU share the buffer and race."""
        self._check_step(q, k_new, v_new, out, ext_score)
        _check(self._lib.kvpop_decode_step_noalloc(self.handle, layer, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(out),
                                             _ptr(ext_score), _stream_ptr(stream)), "kvpop_decode_step_noalloc")

    def prefill_attention_workspace_bytes(self, n_tokens: int) -> int:
        out = ctypes.c_size_t()
        _check(self._lib.kvpop_prefill_attention_workspace_bytes(self.handle, n_tokens, ctypes.byref(out)),
               "kvpop_prefill_attention_workspace_bytes")
        return out.value

    def prefill_attention(self, layer: int, q, k, v, out, lse=None, workspace=None, ext_scores=None, stream=None):
        """Attention outputs of every prompt position under the running top-k
        mask.  q, out: [b][Hq][n][d]; k, v: [b][Hkv][n][d]; lse: optional fp32
        [b][Hq][n]; workspace: a uint8 device tensor of at least
        prefill_attention_workspace_bytes(n) bytes, 16-byte aligned (its first
        units * n int32 are the running cutoffs afterwards).  Does not touch
        the cache."""
        n = self._check_prompt(q, k, v, out, lse, workspace, ext_scores)
        _check(self._lib.kvpop_prefill_attention(self.handle, layer, _ptr(q), _ptr(k), _ptr(v), n, _ptr(ext_scores),
                                           _ptr(out), _ptr(lse), _ptr(workspace),
                                           int(workspace.numel() * workspace.element_size()) if workspace is not None
                                           else 0, _stream_ptr(stream)), "kvpop_prefill_attention")

    def prefill_attention_from_cutoffs(self, layer: int, q, k, v, out, lse=None, workspace=None, stream=None):
        """The attention stage alone, from the cutoffs a previous
        prefill_attention call of the same prompt left in `workspace`."""
        n = self._check_prompt(q, k, v, out, lse, workspace, None)
        _check(self._lib.kvpop_prefill_attention_from_cutoffs(
            self.handle, layer, _ptr(q), _ptr(k), _ptr(v), n, _ptr(out), _ptr(lse), _ptr(workspace),
            int(workspace.numel() * workspace.element_size()) if workspace is not None else 0, _stream_ptr(stream)),
            "kvpop_prefill_attention_from_cutoffs")

    def prefill_with_attention(self, layer: int, q, k, v, out, lse=None, workspace=None, ext_scores=None,
                               stream=None):
        """prefill (whole prompt, empty layer) and prefill_attention in one
        call: the prompt is scored once; afterwards the layer holds the cache
        kvpop_prefill would build and is ready for decode steps."""
        n = self._check_prompt(q, k, v, out, lse, workspace, ext_scores)
        _check(self._lib.kvpop_prefill_with_attention(self.handle, layer, _ptr(q), _ptr(k), _ptr(v), n, _ptr(ext_scores),
                                                _ptr(out), _ptr(lse), _ptr(workspace),
                                                int(workspace.numel() * workspace.element_size())
                                                if workspace is not None else 0, _stream_ptr(stream)),
               "kvpop_prefill_with_attention")

    def _check_prompt(self, q, k, v, out, lse, workspace, ext_scores) -> int:
        import torch
        b, hq, hkv, d = self._dims()
        n = int(k.shape[2]) if isinstance(k, torch.Tensor) and k.dim() == 4 else -1
        self._elems("k", k, (b, hkv, n, d))
        self._elems("v", v, (b, hkv, n, d))
        self._elems("q", q, (b, hq, n, d))
        self._elems("out", out, (b, hq, n, d))
        if lse is not None:
            self._f32("lse", lse, (b, hq, n))
        if ext_scores is not None:
            self._f32("ext_scores", ext_scores, (b, hkv, n))
        if workspace is not None:
            check_tensor(workspace, "workspace", (workspace.numel(),), torch.uint8, self.device)
        return n

    def decode_append(self, layer: int, k_new, v_new, ext_score=None, stream=None):
        b, _, hkv, d = self._dims()
        self._elems("k_new", k_new, (b, hkv, d))
        self._elems("v_new", v_new, (b, hkv, d))
        if ext_score is not None:
            self._f32("ext_score", ext_score, (b, hkv))
        _check(self._lib.kvpop_decode_append(self.handle, layer, _ptr(k_new), _ptr(v_new), _ptr(ext_score),
                                       _stream_ptr(stream)), "kvpop_decode_append")

    def decode_attend(self, layer: int, q, out, stream=None):
        b, hq, _, d = self._dims()
        self._elems("q", q, (b, hq, d))
        self._elems("out", out, (b, hq, d))
        _check(self._lib.kvpop_decode_attend(self.handle, layer, _ptr(q), _ptr(out), _stream_ptr(stream)),
               "kvpop_decode_attend")

    def inspect(self, layer: int, stream=None):
        import numpy as np
        lay = self.layout()
        n = lay.units * lay.slots_per_unit
        pos = np.empty(n, np.int32)
        score = np.empty(n, np.float32)
        state = np.empty(lay.units * 4, np.int32)
        _check(self._lib.kvpop_inspect(self.handle, layer, pos.ctypes.data, score.ctypes.data, state.ctypes.data,
                                 _stream_ptr(stream)), "kvpop_inspect")
        return (pos.reshape(lay.units, lay.slots_per_unit), score.reshape(lay.units, lay.slots_per_unit),
                state.reshape(lay.units, 4))

    def layout(self) -> kvpop_layout_info:
        info = kvpop_layout_info()
        _check(self._lib.kvpop_get_layout(self.handle, ctypes.byref(info)), "kvpop_get_layout")
        return info

    def kv_rows(self, layer: int):
        """View of layer `layer`'s cache rows as a byte tensor [units][slots][row_bytes]."""
        lay = self.layout()
        start = self._off + lay.kv_offset + layer * lay.kv_layer_stride
        n = lay.units * lay.slots_per_unit * lay.row_bytes
        return self.buffer[start:start + n].view(lay.units, lay.slots_per_unit, lay.row_bytes)

    def get_error(self):
        bits = ctypes.c_int32(0)
        st = self._lib.kvpop_get_error(self.handle, ctypes.byref(bits))
        return st, bits.value

    def clear_error(self, stream=None):
        _check(self._lib.kvpop_clear_error(self.handle, _stream_ptr(stream)), "kvpop_clear_error")

    def poison_error(self, bits: int, stream=None):
        _check(self._lib.kvpop_debug_poison_error(self.handle, bits, _stream_ptr(stream)), "kvpop_debug_poison_error")

    def set_test_hook(self, hook: int):
        """Failure injection of a KVPOP_TEST_HOOKS build (kvpop_debug_set_hook)."""
        _check(self._lib.kvpop_debug_set_hook(self.handle, hook), "kvpop_debug_set_hook")
