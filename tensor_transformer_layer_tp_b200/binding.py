"""ctypes binding of libtplayer.so (include/tplayer.h).

Argument marshalling only: torch tensors are turned into device pointers and
the current CUDA stream; every step of the computation runs in the library's
CUDA kernels.  If the library is missing it is built in-tree with nvcc; if that
is impossible, importing fails loudly -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtplayer.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "tplayer.h")
MAX_PARTITIONS = 8

TP_OK, TP_ERR_INVALID_ARG, TP_ERR_UNSUPPORTED, TP_ERR_WORKSPACE, TP_ERR_CUDA, TP_ERR_TIMEOUT = range(6)


class TPError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def _load() -> ctypes.CDLL:
    from . import build as _build
    if not os.path.exists(LIB_PATH) or _build.needs_build():
        _build.build()
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libtplayer.so not found at {LIB_PATH}")
    return ctypes.CDLL(LIB_PATH)


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = _load()
        _declare(_lib)
    return _lib


class tp_layer_dims(ctypes.Structure):
    _fields_ = [("t", ctypes.c_int), ("batch", ctypes.c_int), ("seq", ctypes.c_int),
                ("hidden", ctypes.c_int), ("heads", ctypes.c_int), ("ffn", ctypes.c_int),
                ("causal", ctypes.c_int), ("ln_eps", ctypes.c_float),
                ("dropout_attn", ctypes.c_float), ("dropout_hidden", ctypes.c_float),
                ("seed", ctypes.c_ulonglong), ("recompute", ctypes.c_int)]


_P = ctypes.c_void_p
_PA = _P * MAX_PARTITIONS


class tp_layer_weights(ctypes.Structure):
    _fields_ = [("ln1_g", _P), ("ln1_b", _P), ("w_qkv", _PA), ("b_qkv", _PA), ("w_o", _PA),
                ("b_o", _P), ("ln2_g", _P), ("ln2_b", _P), ("w_fc1", _PA), ("b_fc1", _PA),
                ("w_fc2", _PA), ("b_fc2", _P)]


class tp_layer_grads(tp_layer_weights):
    pass


def _declare(L):
    L.tp_layer_saved_bytes.restype = ctypes.c_size_t
    L.tp_layer_saved_bytes.argtypes = [ctypes.POINTER(tp_layer_dims)]
    L.tp_layer_workspace_bytes.restype = ctypes.c_size_t
    L.tp_layer_workspace_bytes.argtypes = [ctypes.POINTER(tp_layer_dims)]
    L.tp_layer_forward_workspace_bytes.restype = ctypes.c_size_t
    L.tp_layer_forward_workspace_bytes.argtypes = [ctypes.POINTER(tp_layer_dims)]
    L.tp_layer_forward.restype = ctypes.c_int
    L.tp_layer_forward.argtypes = [ctypes.POINTER(tp_layer_dims), ctypes.POINTER(tp_layer_weights),
                                   _P, _P, _P, _P, ctypes.c_size_t, _P, ctypes.c_size_t, _P]
    L.tp_layer_backward.restype = ctypes.c_int
    L.tp_layer_backward.argtypes = [ctypes.POINTER(tp_layer_dims), ctypes.POINTER(tp_layer_weights),
                                    _P, _P, _P, ctypes.c_size_t, _P, _P,
                                    ctypes.POINTER(tp_layer_grads), _P, ctypes.c_size_t, _P]
    L.tp_layer_rank_saved_bytes.restype = ctypes.c_size_t
    L.tp_layer_rank_saved_bytes.argtypes = [ctypes.POINTER(tp_layer_dims)]
    L.tp_layer_rank_workspace_bytes.restype = ctypes.c_size_t
    L.tp_layer_rank_workspace_bytes.argtypes = [ctypes.POINTER(tp_layer_dims)]
    L.tp_layer_rank_forward.restype = ctypes.c_int
    L.tp_layer_rank_forward.argtypes = [ctypes.POINTER(tp_layer_dims), ctypes.c_int, ctypes.c_int,
                                        ctypes.POINTER(tp_layer_weights), _P, _P, _P, _P, _P,
                                        ctypes.c_size_t, _P]
    L.tp_layer_rank_backward.restype = ctypes.c_int
    L.tp_layer_rank_backward.argtypes = [ctypes.POINTER(tp_layer_dims), ctypes.c_int, ctypes.c_int,
                                         ctypes.POINTER(tp_layer_weights), _P, _P, _P, ctypes.c_size_t,
                                         _P, _P, _P, ctypes.POINTER(tp_layer_grads), _P,
                                         ctypes.c_size_t, _P]
    L.tp_xent_rank_workspace_bytes.restype = ctypes.c_size_t
    L.tp_xent_rank_workspace_bytes.argtypes = [ctypes.c_int] * 4
    L.vocab_parallel_xent_rank.restype = ctypes.c_int
    L.vocab_parallel_xent_rank.argtypes = [ctypes.c_int] * 6 + [_P, _P, _P, _P, _P, _P, _P, _P, _P,
                                                                ctypes.c_size_t, _P]
    L.tp_xent_workspace_bytes.restype = ctypes.c_size_t
    L.tp_xent_workspace_bytes.argtypes = [ctypes.c_int] * 4
    L.vocab_parallel_xent.restype = ctypes.c_int
    L.vocab_parallel_xent.argtypes = [ctypes.c_int] * 4 + [_P, ctypes.POINTER(_P), _P, _P, _P, _P,
                                                           ctypes.POINTER(_P), _P, ctypes.c_size_t, _P]
    L.tp_xent_forward_workspace_bytes.restype = ctypes.c_size_t
    L.tp_xent_forward_workspace_bytes.argtypes = [ctypes.c_int] * 4
    L.tp_xent_explicit_workspace_bytes.restype = ctypes.c_size_t
    L.tp_xent_explicit_workspace_bytes.argtypes = [ctypes.c_int] * 4
    L.vocab_parallel_xent_explicit.restype = ctypes.c_int
    L.vocab_parallel_xent_explicit.argtypes = L.vocab_parallel_xent.argtypes
    L.vocab_parallel_xent_static.restype = ctypes.c_int
    L.vocab_parallel_xent_static.argtypes = [ctypes.c_int] * 4 + [_P, ctypes.POINTER(_P), _P, _P, _P,
                                                                  _P, ctypes.POINTER(_P), _P]
    L.vocab_parallel_embedding_forward.restype = ctypes.c_int
    L.vocab_parallel_embedding_forward.argtypes = [ctypes.c_int] * 4 + [_P, ctypes.POINTER(_P), _P, _P]
    L.tp_embedding_backward_workspace_bytes.restype = ctypes.c_size_t
    L.tp_embedding_backward_workspace_bytes.argtypes = [ctypes.c_int] * 4
    L.vocab_parallel_embedding_backward.restype = ctypes.c_int
    L.vocab_parallel_embedding_backward.argtypes = [ctypes.c_int] * 4 + [
        _P, _P, ctypes.POINTER(_P), ctypes.c_int, _P, ctypes.c_size_t, _P]
    L.tp_gemm.restype = ctypes.c_int
    L.tp_gemm.argtypes = [ctypes.c_int] * 5 + [ctypes.POINTER(_P), ctypes.c_int, ctypes.POINTER(_P),
                                               ctypes.c_int, ctypes.POINTER(_P), ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int, _P]
    L.tp_profile_enable.restype = ctypes.c_int
    L.tp_profile_enable.argtypes = [ctypes.c_int]
    L.tp_profile_reset.restype = ctypes.c_int
    L.tp_profile_reset.argtypes = []
    L.tp_selftest_wait_timeout.restype = ctypes.c_int
    L.tp_selftest_wait_timeout.argtypes = [_P]
    L.tp_partition_sum.restype = ctypes.c_int
    L.tp_partition_sum.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, ctypes.c_longlong,
                                   _P, _P, _P, _P]
    L.tp_gelu_eval.restype = ctypes.c_int
    L.tp_gelu_eval.argtypes = [ctypes.c_int, _P, _P, _P, _P]
    L.tp_profile_record.restype = ctypes.c_int
    L.tp_profile_record.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_int),
                                    ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_double)]
    L.tp_profile_summary.restype = ctypes.c_int
    L.tp_profile_summary.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_int),
                                     ctypes.POINTER(ctypes.c_double)]
    L.tp_device_status.restype = ctypes.c_int
    L.tp_device_status.argtypes = [_P]
    L.tp_status_string.restype = ctypes.c_char_p
    L.tp_status_string.argtypes = [ctypes.c_int]


def header_functions() -> list:
    """Names of the functions include/tplayer.h declares."""
    text = open(HEADER_PATH).read()
    return re.findall(r"^TP_API\s+[\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M)


def status_string(status: int) -> str:
    return lib().tp_status_string(int(status)).decode()


# --------------------------------------------------------------------- helpers

def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(status: int, where: str):
    if status != TP_OK:
        raise TPError(status, where)


def make_dims(t, batch, seq, hidden, heads, ffn, causal=True, ln_eps=1e-5, dropout_attn=0.0,
              dropout_hidden=0.0, seed=0, recompute=False) -> tp_layer_dims:
    return tp_layer_dims(t, batch, seq, hidden, heads, ffn, int(bool(causal)), float(ln_eps),
                         float(dropout_attn), float(dropout_hidden), int(seed), int(bool(recompute)))


def _fill(struct_type, p: dict, t: int):
    s = struct_type()
    for name in ("ln1_g", "ln1_b", "b_o", "ln2_g", "ln2_b", "b_fc2"):
        setattr(s, name, _ptr(p[name]))
    for name in ("w_qkv", "b_qkv", "w_o", "w_fc1", "b_fc1", "w_fc2"):
        arr = getattr(s, name)
        for i in range(t):
            arr[i] = _ptr(p[name][i])
    return s


# --------------------------------------------------------------------- entry points

def tp_layer_saved_bytes(dims: tp_layer_dims) -> int:
    return int(lib().tp_layer_saved_bytes(ctypes.byref(dims)))


def tp_layer_workspace_bytes(dims: tp_layer_dims) -> int:
    return int(lib().tp_layer_workspace_bytes(ctypes.byref(dims)))


def tp_layer_forward_workspace_bytes(dims: tp_layer_dims) -> int:
    return int(lib().tp_layer_forward_workspace_bytes(ctypes.byref(dims)))


def _nbytes(t):
    return t.numel() * t.element_size()


def tp_layer_forward(dims, weights: dict, x, valid_len, y, saved, stream=None, ws=None):
    w = _fill(tp_layer_weights, weights, dims.t)
    _check(lib().tp_layer_forward(ctypes.byref(dims), ctypes.byref(w), _ptr(x), _ptr(valid_len),
                                  _ptr(y), _ptr(saved), _nbytes(saved), _ptr(ws),
                                  _nbytes(ws) if ws is not None else 0, _stream(stream)),
           "tp_layer_forward")


def tp_layer_backward(dims, weights: dict, x, valid_len, saved, dy, dx, grads: dict, ws,
                      stream=None):
    w = _fill(tp_layer_weights, weights, dims.t)
    g = _fill(tp_layer_grads, grads, dims.t)
    _check(lib().tp_layer_backward(ctypes.byref(dims), ctypes.byref(w), _ptr(x), _ptr(valid_len),
                                   _ptr(saved), _nbytes(saved), _ptr(dy), _ptr(dx), ctypes.byref(g),
                                   _ptr(ws), _nbytes(ws), _stream(stream)),
           "tp_layer_backward")


def tp_layer_rank_saved_bytes(dims: tp_layer_dims) -> int:
    return int(lib().tp_layer_rank_saved_bytes(ctypes.byref(dims)))


def tp_layer_rank_workspace_bytes(dims: tp_layer_dims) -> int:
    return int(lib().tp_layer_rank_workspace_bytes(ctypes.byref(dims)))


def tp_layer_rank_forward(dims, rank, segment, weights: dict, x, valid_len, partial, y, saved,
                          stream=None):
    """One segment of partition `rank`'s forward; `weights` holds the rank's
    partitioned tensors as one-element lists and the replicated ones whole."""
    w = _fill(tp_layer_weights, weights, 1)
    _check(lib().tp_layer_rank_forward(ctypes.byref(dims), rank, segment, ctypes.byref(w), _ptr(x),
                                       _ptr(valid_len), _ptr(partial), _ptr(y), _ptr(saved),
                                       _nbytes(saved), _stream(stream)),
           "tp_layer_rank_forward")


def tp_layer_rank_backward(dims, rank, segment, weights: dict, x, valid_len, saved, dy, partial, dx,
                           grads: dict, ws, stream=None):
    w = _fill(tp_layer_weights, weights, 1)
    g = _fill(tp_layer_grads, grads, 1)
    _check(lib().tp_layer_rank_backward(ctypes.byref(dims), rank, segment, ctypes.byref(w), _ptr(x),
                                        _ptr(valid_len), _ptr(saved), _nbytes(saved), _ptr(dy),
                                        _ptr(partial), _ptr(dx), ctypes.byref(g), _ptr(ws), _nbytes(ws),
                                        _stream(stream)),
           "tp_layer_rank_backward")


def tp_xent_rank_workspace_bytes(t, tokens, hidden, vocab) -> int:
    return int(lib().tp_xent_rank_workspace_bytes(t, tokens, hidden, vocab))


def vocab_parallel_xent_rank(t, rank, segment, tokens, hidden, vocab, x, emb, target, comm, loss=None,
                             loss_per_token=None, dx=None, demb=None, ws=None, stream=None):
    """One segment of vocab partition `rank`'s loss (include/tplayer.h)."""
    _check(lib().vocab_parallel_xent_rank(t, rank, segment, tokens, hidden, vocab, _ptr(x), _ptr(emb),
                                          _ptr(target), _ptr(comm), _ptr(loss), _ptr(loss_per_token),
                                          _ptr(dx), _ptr(demb), _ptr(ws), _nbytes(ws), _stream(stream)),
           "vocab_parallel_xent_rank")


def tp_xent_workspace_bytes(t, tokens, hidden, vocab) -> int:
    return int(lib().tp_xent_workspace_bytes(t, tokens, hidden, vocab))


def tp_xent_forward_workspace_bytes(t, tokens, hidden, vocab) -> int:
    return int(lib().tp_xent_forward_workspace_bytes(t, tokens, hidden, vocab))


def tp_xent_explicit_workspace_bytes(t, tokens, hidden, vocab) -> int:
    return int(lib().tp_xent_explicit_workspace_bytes(t, tokens, hidden, vocab))


def vocab_parallel_xent(t, tokens, hidden, vocab, x, emb: list, target, loss, loss_per_token=None,
                        dx=None, demb=None, ws=None, stream=None, explicit=False):
    """The fused loss (explicit=False) or its step-by-step fp32-logit form."""
    emb_arr = (_P * t)(*[_ptr(e) for e in emb])
    demb_arr = (_P * t)(*[_ptr(e) for e in demb]) if demb is not None else None
    fn = lib().vocab_parallel_xent_explicit if explicit else lib().vocab_parallel_xent
    _check(fn(t, tokens, hidden, vocab, _ptr(x), emb_arr, _ptr(target), _ptr(loss),
              _ptr(loss_per_token), _ptr(dx), demb_arr, _ptr(ws), ws.numel() * ws.element_size(),
              _stream(stream)),
           "vocab_parallel_xent_explicit" if explicit else "vocab_parallel_xent")


XENT_STATIC_SCRATCH_BYTES = 64 << 20


def vocab_parallel_xent_static(t, tokens, hidden, vocab, x, emb: list, target, loss,
                               loss_per_token=None, dx=None, demb=None, stream=None):
    """vocab_parallel_xent without a caller workspace: the library's fixed scratch is used."""
    emb_arr = (_P * t)(*[_ptr(e) for e in emb])
    demb_arr = (_P * t)(*[_ptr(e) for e in demb]) if demb is not None else None
    _check(lib().vocab_parallel_xent_static(t, tokens, hidden, vocab, _ptr(x), emb_arr, _ptr(target),
                                            _ptr(loss), _ptr(loss_per_token), _ptr(dx), demb_arr,
                                            _stream(stream)),
           "vocab_parallel_xent_static")


def vocab_parallel_embedding_forward(t, tokens, hidden, vocab, ids, emb: list, out, stream=None):
    emb_arr = (_P * t)(*[_ptr(e) for e in emb])
    _check(lib().vocab_parallel_embedding_forward(t, tokens, hidden, vocab, _ptr(ids), emb_arr,
                                                  _ptr(out), _stream(stream)),
           "vocab_parallel_embedding_forward")


def tp_embedding_backward_workspace_bytes(t, tokens, hidden, vocab) -> int:
    return int(lib().tp_embedding_backward_workspace_bytes(t, tokens, hidden, vocab))


def vocab_parallel_embedding_backward(t, tokens, hidden, vocab, ids, dout, demb: list, accumulate,
                                      ws, stream=None):
    demb_arr = (_P * t)(*[_ptr(e) for e in demb])
    _check(lib().vocab_parallel_embedding_backward(t, tokens, hidden, vocab, _ptr(ids), _ptr(dout),
                                                   demb_arr, int(bool(accumulate)), _ptr(ws),
                                                   _nbytes(ws), _stream(stream)),
           "vocab_parallel_embedding_backward")


def tp_gemm(groups, sum_groups, m, n, k, a: list, a_layout, b: list, b_layout, c: list, c_fp32,
            tile_n=0, cta_pair=-1, stream=None):
    A = (_P * len(a))(*[_ptr(v) for v in a])
    B = (_P * len(b))(*[_ptr(v) for v in b])
    C = (_P * len(c))(*[_ptr(v) for v in c])
    _check(lib().tp_gemm(groups, sum_groups, m, n, k, A, a_layout, B, b_layout, C, c_fp32,
                         tile_n, cta_pair, _stream(stream)), "tp_gemm")


def tp_partition_sum(partials: list, out, bias=None, residual=None, stream=None):
    """out = bf16(sum_g partials[g] + bias + residual); partials: fp32 [rows, cols] tensors."""
    rows, cols = partials[0].shape
    P = (_P * len(partials))(*[_ptr(v) for v in partials])
    _check(lib().tp_partition_sum(len(partials), rows, cols, P, partials[0].stride(0), _ptr(bias),
                                  _ptr(residual), _ptr(out), _stream(stream)), "tp_partition_sum")


def tp_gelu_eval(x, gelu=None, dgelu=None, stream=None):
    """gelu[i] = GeLU(x[i]), dgelu[i] = GeLU'(x[i]) on the device (fp32 tensors)."""
    _check(lib().tp_gelu_eval(int(x.numel()), _ptr(x), _ptr(gelu) if gelu is not None else None,
                              _ptr(dgelu) if dgelu is not None else None, _stream(stream)),
           "tp_gelu_eval")


KERNEL_CLASSES = ("gemm", "attn_fwd", "attn_bwd", "ln_fwd", "ln_bwd", "reduce", "xent_stats",
                  "xent_combine", "xent_grad", "elementwise")


def tp_profile_enable(max_records: int):
    _check(lib().tp_profile_enable(int(max_records)), "tp_profile_enable")


def tp_profile_reset():
    _check(lib().tp_profile_reset(), "tp_profile_reset")


def tp_profile_summary() -> dict:
    """{class name: (kernels launched, summed device ms)} for the records taken."""
    out = {}
    for i, name in enumerate(KERNEL_CLASSES):
        k, ms = ctypes.c_int(0), ctypes.c_double(0.0)
        _check(lib().tp_profile_summary(i, ctypes.byref(k), ctypes.byref(ms)), "tp_profile_summary")
        out[name] = (k.value, ms.value)
    return out


def tp_profile_records() -> list:
    """[(class name, kernels, device ms)] per recorded launch, in enqueue order."""
    out = []
    i = 0
    kind, k, ms = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_double(0.0)
    while lib().tp_profile_record(i, ctypes.byref(kind), ctypes.byref(k), ctypes.byref(ms)) == TP_OK:
        out.append((KERNEL_CLASSES[kind.value], k.value, ms.value))
        i += 1
    return out


def tp_selftest_wait_timeout(stream=None):
    """Enqueue the bounded-wait self-test kernel (see include/tplayer.h)."""
    _check(lib().tp_selftest_wait_timeout(_stream(stream)), "tp_selftest_wait_timeout")


def tp_device_status(stream=None):
    _check(lib().tp_device_status(_stream(stream)), "tp_device_status")
