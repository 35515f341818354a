"""ctypes binding of liblisa.so (the C ABI declared in include/lisa.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors (device memory and streams come from
PyTorch); the functions take the same names and arguments as the C entry
points.  There is no fallback: if the library is missing, importing this module
raises.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblisa.so")

LISA_OK = 0
LISA_ERR_INVALID_ARG = 1
LISA_ERR_UNSUPPORTED = 2
LISA_ERR_CUDA = 3
LISA_ERR_WORKSPACE = 4
LISA_BF16 = 0
LISA_FP32 = 1
LISA_DEVERR_POS = 1
LISA_DEVERR_TIMEOUT = 2
LISA_DEVERR_CHECK = 4
LISA_DEBUG_FORCE_TIMEOUT = 1
LISA_OP_DECODE = 0
LISA_OP_PREFILL = 1
LISA_OP_INDEXER_TOPK = 2
LISA_OP_PREFILL_WINDOW = 3
LISA_VAR_KEY_PER_INDEXER_HEAD = 1
LISA_VAR_SHARED_SET = 2
LISA_VAR_LINEAR_KV_PER_QUERY_HEAD = 4

EXPORTED = [
    "lisa_workspace_bytes",
    "lisa_append_cache",
    "lisa_indexer_topk",
    "lisa_indexer_topk_noalloc",
    "lisa_decode_step",
    "lisa_prefill",
    "lisa_decode_step_window",
    "lisa_prefill_window",
    "lisa_indexer_kl",
    "lisa_workspace_bytes_variant",
    "lisa_append_cache_variant",
    "lisa_indexer_topk_variant",
    "lisa_decode_step_variant",
    "lisa_prefill_variant",
    "lisa_project_in",
    "lisa_project_out",
    "lisa_status_str",
    "lisa_last_error_msg",
    "lisa_version",
]


class LisaLayerC(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("d", ctypes.c_int),
        ("HI", ctypes.c_int), ("dI", ctypes.c_int), ("M", ctypes.c_int), ("L_max", ctypes.c_int),
        ("dtype", ctypes.c_int),
        ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p), ("kidx_cache", ctypes.c_void_p),
        ("state", ctypes.c_void_p), ("pos", ctypes.c_void_p), ("err_word", ctypes.c_void_p),
        ("decode_split", ctypes.c_int), ("independent", ctypes.c_int), ("debug_flags", ctypes.c_int),
    ]


class LisaProjC(ctypes.Structure):
    _fields_ = [("Hm", ctypes.c_int), ("W_in", ctypes.c_void_p), ("W_o", ctypes.c_void_p)]


class LisaError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{status_str(status)}: {msg}")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} not built: run `python -m hybrid_linear_top_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    L = ctypes.POINTER(LisaLayerC)
    lib.lisa_workspace_bytes.argtypes = [L, ctypes.c_int, ctypes.c_int]
    lib.lisa_workspace_bytes.restype = ctypes.c_size_t
    lib.lisa_append_cache.argtypes = [L, P, P, P, ctypes.c_int, P]
    lib.lisa_append_cache.restype = ctypes.c_int
    lib.lisa_indexer_topk.argtypes = [L, P, P, ctypes.c_int, P, P, ctypes.c_size_t, P]
    lib.lisa_indexer_topk.restype = ctypes.c_int
    lib.lisa_indexer_topk_noalloc.argtypes = [L, P, P, ctypes.c_int, P, P]
    lib.lisa_indexer_topk_noalloc.restype = ctypes.c_int
    lib.lisa_decode_step.argtypes = [L, P, P, P, P, P, P, P, ctypes.c_int, P, P, P, ctypes.c_size_t, P]
    lib.lisa_decode_step.restype = ctypes.c_int
    lib.lisa_prefill.argtypes = [L, ctypes.c_int, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    lib.lisa_prefill.restype = ctypes.c_int
    lib.lisa_decode_step_window.argtypes = [L, P, P, P, P, P, ctypes.c_int, P, P, P]
    lib.lisa_decode_step_window.restype = ctypes.c_int
    lib.lisa_prefill_window.argtypes = [L, ctypes.c_int, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    lib.lisa_prefill_window.restype = ctypes.c_int
    lib.lisa_indexer_kl.argtypes = [L, ctypes.c_int, P, P, P, P, P]
    lib.lisa_indexer_kl.restype = ctypes.c_int
    I = ctypes.c_int
    lib.lisa_workspace_bytes_variant.argtypes = [L, I, I, I]
    lib.lisa_workspace_bytes_variant.restype = ctypes.c_size_t
    lib.lisa_append_cache_variant.argtypes = [L, I, P, P, P, I, P]
    lib.lisa_append_cache_variant.restype = I
    lib.lisa_indexer_topk_variant.argtypes = [L, I, P, P, I, P, P, ctypes.c_size_t, P]
    lib.lisa_indexer_topk_variant.restype = I
    lib.lisa_decode_step_variant.argtypes = [L, I, P, P, P, P, P, P, P, P, P, I, P, P, P, ctypes.c_size_t, P]
    lib.lisa_decode_step_variant.restype = I
    lib.lisa_prefill_variant.argtypes = [L, I, I, P, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    lib.lisa_prefill_variant.restype = I
    PJ = ctypes.POINTER(LisaProjC)
    lib.lisa_project_in.argtypes = [L, I, PJ, I, P, P, P, P, P, P, P, P, P]
    lib.lisa_project_in.restype = I
    lib.lisa_project_out.argtypes = [L, PJ, I, P, P, P]
    lib.lisa_project_out.restype = I
    lib.lisa_status_str.argtypes = [ctypes.c_int]
    lib.lisa_status_str.restype = ctypes.c_char_p
    lib.lisa_last_error_msg.argtypes = []
    lib.lisa_last_error_msg.restype = ctypes.c_char_p
    lib.lisa_version.argtypes = []
    lib.lisa_version.restype = ctypes.c_char_p
    return lib


_lib = _load()


def lib():
    return _lib


def status_str(s):
    return _lib.lisa_status_str(int(s)).decode()


def last_error_msg():
    return _lib.lisa_last_error_msg().decode()


def version():
    return _lib.lisa_version().decode()


def _ptr(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status):
    if status != LISA_OK:
        raise LisaError(status, last_error_msg())


TORCH_DTYPE = {LISA_BF16: torch.bfloat16, LISA_FP32: torch.float32}


class Layer:
    """Geometry and caller-owned buffers of one LISA layer (a lisa_layer).

    k_cache, v_cache [B, Hkv, L_max, d]; kidx_cache [B, Hkv, L_max, dI] in the
    storage dtype; state [B, Hq, d, d] fp32; pos [B] int32; err_word [1] int32
    (all on one CUDA device).  decode_split: CTAs per (sequence, KV head) of
    the decode step (0 = the library's choice, or 4, 8, 16).  independent: 1
    declares the layer's decode steps independent of the launch before them on
    the stream (no wait for it).  debug_flags: LISA_DEBUG_* bits."""

    def __init__(self, B, Hq, Hkv, d, HI, dI, M, L_max, dtype, k_cache, v_cache, kidx_cache, state, pos,
                 err_word=None, decode_split=0, independent=0, debug_flags=0):
        self.B, self.Hq, self.Hkv, self.d, self.HI, self.dI, self.M, self.L_max = B, Hq, Hkv, d, HI, dI, M, L_max
        self.dtype = dtype
        self.k_cache, self.v_cache, self.kidx_cache = k_cache, v_cache, kidx_cache
        self.state, self.pos, self.err_word = state, pos, err_word
        self.decode_split = decode_split
        self.independent = independent
        self.debug_flags = debug_flags

    @classmethod
    def allocate(cls, B, Hq, Hkv, d, HI, dI, M, L_max, dtype=LISA_BF16, device="cuda", decode_split=0):
        tdt = TORCH_DTYPE[dtype]
        return cls(B, Hq, Hkv, d, HI, dI, M, L_max, dtype,
                   torch.zeros(B, Hkv, L_max, d, dtype=tdt, device=device),
                   torch.zeros(B, Hkv, L_max, d, dtype=tdt, device=device),
                   torch.zeros(B, Hkv, L_max, dI, dtype=tdt, device=device),
                   torch.zeros(B, Hq, d, d, dtype=torch.float32, device=device),
                   torch.zeros(B, dtype=torch.int32, device=device),
                   torch.zeros(1, dtype=torch.int32, device=device), decode_split)

    def c_struct(self):
        return LisaLayerC(
            self.B, self.Hq, self.Hkv, self.d, self.HI, self.dI, self.M, self.L_max, self.dtype,
            _ptr(self.k_cache), _ptr(self.v_cache), _ptr(self.kidx_cache), _ptr(self.state), _ptr(self.pos),
            _ptr(self.err_word), int(self.decode_split), int(self.independent), int(self.debug_flags),
        )

    @property
    def torch_dtype(self):
        return TORCH_DTYPE[self.dtype]


def lisa_workspace_bytes(layer, T, op):
    c = layer.c_struct() if isinstance(layer, Layer) else layer
    return int(_lib.lisa_workspace_bytes(ctypes.byref(c), int(T), int(op)))


def alloc_workspace(layer, T, op, device="cuda"):
    """Workspace for `op` (zero-filled: the decode step's workspace must start
    at zero, and every call leaves it ready for the next)."""
    n = lisa_workspace_bytes(layer, T, op)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device)


def lisa_append_cache(layer, k, v, kidx, T, stream=None):
    c = layer.c_struct()
    _check(_lib.lisa_append_cache(ctypes.byref(c), _ptr(k), _ptr(v), _ptr(kidx), int(T), _stream(stream)))


def lisa_indexer_topk(layer, qidx, w, T, idx_out, workspace, stream=None):
    c = layer.c_struct()
    _check(_lib.lisa_indexer_topk(ctypes.byref(c), _ptr(qidx), _ptr(w), int(T), _ptr(idx_out), _ptr(workspace),
                                  workspace.numel() if workspace is not None else 0, _stream(stream)))


def lisa_indexer_topk_noalloc(layer, qidx, w, T, idx_out, stream=None):
    c = layer.c_struct()
    _check(_lib.lisa_indexer_topk_noalloc(ctypes.byref(c), _ptr(qidx), _ptr(w), int(T), _ptr(idx_out),
                                          _stream(stream)))


NOALLOC_SCRATCH_BYTES = 16 << 20


def lisa_decode_step(layer, q, k, v, kidx, qidx, w, gate_logit, fuse_append, out, idx_out, workspace,
                     stream=None):
    c = layer.c_struct()
    _check(_lib.lisa_decode_step(ctypes.byref(c), _ptr(q), _ptr(k), _ptr(v), _ptr(kidx), _ptr(qidx), _ptr(w),
                                 _ptr(gate_logit), int(bool(fuse_append)), _ptr(out), _ptr(idx_out),
                                 _ptr(workspace), workspace.numel() if workspace is not None else 0,
                                 _stream(stream)))


def lisa_decode_step_window(layer, q, k, v, kidx, gate_logit, fuse_append, out, idx_out, stream=None):
    c = layer.c_struct()
    _check(_lib.lisa_decode_step_window(ctypes.byref(c), _ptr(q), _ptr(k), _ptr(v), _ptr(kidx), _ptr(gate_logit),
                                        int(bool(fuse_append)), _ptr(out), _ptr(idx_out), _stream(stream)))


def lisa_prefill_window(layer, T, q, k, v, kidx, gate_logit, out, idx_out, workspace, stream=None):
    c = layer.c_struct()
    _check(_lib.lisa_prefill_window(ctypes.byref(c), int(T), _ptr(q), _ptr(k), _ptr(v), _ptr(kidx),
                                    _ptr(gate_logit), _ptr(out), _ptr(idx_out), _ptr(workspace),
                                    workspace.numel() if workspace is not None else 0, _stream(stream)))


def lisa_indexer_kl(layer, T, q, qidx, w, kl_out, stream=None):
    c = layer.c_struct()
    _check(_lib.lisa_indexer_kl(ctypes.byref(c), int(T), _ptr(q), _ptr(qidx), _ptr(w), _ptr(kl_out),
                                _stream(stream)))


def lisa_prefill(layer, T, q, k, v, kidx, qidx, w, gate_logit, out, idx_out, workspace, stream=None):
    c = layer.c_struct()
    _check(_lib.lisa_prefill(ctypes.byref(c), int(T), _ptr(q), _ptr(k), _ptr(v), _ptr(kidx), _ptr(qidx), _ptr(w),
                             _ptr(gate_logit), _ptr(out), _ptr(idx_out), _ptr(workspace),
                             workspace.numel() if workspace is not None else 0, _stream(stream)))


# ---------------------------------------------------------------- definition variants
def variant_planes(layer, variant):
    """(P, Gs): indexer-key planes and selection groups under `variant`."""
    Gs = 1 if variant & LISA_VAR_SHARED_SET else layer.Hkv
    P = layer.HI if variant & LISA_VAR_KEY_PER_INDEXER_HEAD else Gs
    return P, Gs


def lisa_workspace_bytes_variant(layer, variant, T, op):
    c = layer.c_struct() if isinstance(layer, Layer) else layer
    return int(_lib.lisa_workspace_bytes_variant(ctypes.byref(c), int(variant), int(T), int(op)))


def alloc_workspace_variant(layer, variant, T, op, device="cuda"):
    n = lisa_workspace_bytes_variant(layer, variant, T, op)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device)


def lisa_append_cache_variant(layer, variant, k, v, kidx, T, stream=None):
    c = layer.c_struct()
    _check(_lib.lisa_append_cache_variant(ctypes.byref(c), int(variant), _ptr(k), _ptr(v), _ptr(kidx), int(T),
                                          _stream(stream)))


def lisa_indexer_topk_variant(layer, variant, qidx, w, T, idx_out, workspace, stream=None):
    c = layer.c_struct()
    _check(_lib.lisa_indexer_topk_variant(ctypes.byref(c), int(variant), _ptr(qidx), _ptr(w), int(T), _ptr(idx_out),
                                          _ptr(workspace), workspace.numel() if workspace is not None else 0,
                                          _stream(stream)))


def lisa_decode_step_variant(layer, variant, q, k, v, kidx, qidx, w, gate_logit, k_lin, v_lin, fuse_append, out,
                             idx_out, workspace, stream=None):
    c = layer.c_struct()
    _check(_lib.lisa_decode_step_variant(ctypes.byref(c), int(variant), _ptr(q), _ptr(k), _ptr(v), _ptr(kidx),
                                         _ptr(qidx), _ptr(w), _ptr(gate_logit), _ptr(k_lin), _ptr(v_lin),
                                         int(bool(fuse_append)), _ptr(out), _ptr(idx_out), _ptr(workspace),
                                         workspace.numel() if workspace is not None else 0, _stream(stream)))


def lisa_prefill_variant(layer, variant, T, q, k, v, kidx, qidx, w, gate_logit, k_lin, v_lin, out, idx_out,
                         workspace, stream=None):
    c = layer.c_struct()
    _check(_lib.lisa_prefill_variant(ctypes.byref(c), int(variant), int(T), _ptr(q), _ptr(k), _ptr(v), _ptr(kidx),
                                     _ptr(qidx), _ptr(w), _ptr(gate_logit), _ptr(k_lin), _ptr(v_lin), _ptr(out),
                                     _ptr(idx_out), _ptr(workspace),
                                     workspace.numel() if workspace is not None else 0, _stream(stream)))


# ---------------------------------------------------------------- projections
class Proj:
    """Projection weights of one layer (a lisa_proj): W_in [N_in, Hm] and
    W_o [Hm, Hq*d], bf16 CUDA tensors (out-features x in-features)."""

    def __init__(self, Hm, W_in, W_o):
        self.Hm, self.W_in, self.W_o = Hm, W_in, W_o

    def c_struct(self):
        return LisaProjC(int(self.Hm), _ptr(self.W_in), _ptr(self.W_o))


def proj_widths(layer, variant=0):
    """Column widths of the front-end fields q, k, v, qidx, kidx, w, gate_logit."""
    P, _ = variant_planes(layer, variant)
    return (layer.Hq * layer.d, layer.Hkv * layer.d, layer.Hkv * layer.d, layer.HI * layer.dI, P * layer.dI,
            layer.HI, layer.Hq)


def lisa_project_in(layer, variant, proj, T, x, q, k, v, qidx, kidx, w, gate_logit, stream=None):
    c, pj = layer.c_struct(), proj.c_struct()
    _check(_lib.lisa_project_in(ctypes.byref(c), int(variant), ctypes.byref(pj), int(T), _ptr(x), _ptr(q), _ptr(k),
                                _ptr(v), _ptr(qidx), _ptr(kidx), _ptr(w), _ptr(gate_logit), _stream(stream)))


def lisa_project_out(layer, proj, T, o, y, stream=None):
    c, pj = layer.c_struct(), proj.c_struct()
    _check(_lib.lisa_project_out(ctypes.byref(c), ctypes.byref(pj), int(T), _ptr(o), _ptr(y), _stream(stream)))
