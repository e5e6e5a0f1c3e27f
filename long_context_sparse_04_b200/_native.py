"""ctypes binding of libdsa.so (include/dsa.h): argument marshalling only.

Every compute step runs in the CUDA library.  If the library is missing this
module raises on import; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdsa.so")

DSA_OK, DSA_ERR_INVALID_ARG, DSA_ERR_UNSUPPORTED, DSA_ERR_CUDA = 0, 1, 2, 3
DSA_ERR_OUT_OF_RANGE, DSA_ERR_TIMEOUT, DSA_ERR_WORKSPACE = 4, 5, 6
DSA_F32, DSA_BF16, DSA_FP8_E4M3 = 0, 1, 2
DSA_ALGO_AUTO, DSA_ALGO_SIMT, DSA_ALGO_STAGED = 0, 1, 2
DSA_OP_INDEXER, DSA_OP_TOPK, DSA_OP_SPARSE_MLA, DSA_OP_DECODE_STEP, DSA_OP_FORWARD = range(5)
DSA_OP_CACHE_APPEND = 5
DSA_OP_INDEXER_KL, DSA_OP_INDEXER_BACKWARD = 6, 7
DSA_KERNEL_INDEXER_SIMT, DSA_KERNEL_INDEXER_TC, DSA_KERNEL_TOPK = 0x01, 0x02, 0x04
DSA_KERNEL_MLA_SIMT, DSA_KERNEL_MLA_TC, DSA_KERNEL_MLA_COMBINE = 0x08, 0x10, 0x20
DSA_KERNEL_CACHE_APPEND = 0x40
DSA_KERNEL_OUT_PROJ, DSA_KERNEL_OUT_PROJ_REDUCE = 0x80, 0x100
DSA_KERNEL_WARMUP = 0x200
DSA_FAULT_INDEXER_ACC_RELEASE = 0x1


class dsa_dims(ctypes.Structure):
    _fields_ = [("n_idx_heads", ctypes.c_int32), ("d_idx", ctypes.c_int32),
                ("n_heads", ctypes.c_int32), ("d_c", ctypes.c_int32), ("d_r", ctypes.c_int32),
                ("topk", ctypes.c_int32), ("idx_dtype", ctypes.c_int), ("mla_dtype", ctypes.c_int),
                ("sm_scale", ctypes.c_float), ("algo", ctypes.c_int)]


class dsa_rows(ctypes.Structure):
    _fields_ = [("num_rows", ctypes.c_int32), ("row_seq", ctypes.c_void_p),
                ("row_klen", ctypes.c_void_p), ("max_klen", ctypes.c_int32),
                ("q_group", ctypes.c_int32)]


class dsa_cache(ctypes.Structure):
    _fields_ = [("latent", ctypes.c_void_p), ("idx_k", ctypes.c_void_p),
                ("idx_k_scale", ctypes.c_void_p), ("seq_start", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("page_size", ctypes.c_int32),
                ("max_pages_per_seq", ctypes.c_int32), ("num_seqs", ctypes.c_int32),
                ("num_tokens", ctypes.c_int64)]


class dsa_proj_dims(ctypes.Structure):
    _fields_ = [("n_heads", ctypes.c_int32), ("d_c", ctypes.c_int32), ("d_v", ctypes.c_int32),
                ("d_model", ctypes.c_int32)]


_P = ctypes.c_void_p
_SIGS = {
    "dsa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "dsa_last_error": (ctypes.c_char_p, []),
    "dsa_version": (ctypes.c_int32, []),
    "dsa_workspace_size": (ctypes.c_size_t, [_P, _P, ctypes.c_int]),
    "dsa_workspace_init": (ctypes.c_int, [_P, ctypes.c_size_t, _P]),
    "dsa_read_device_status": (ctypes.c_int, [_P, _P, _P, _P]),
    "dsa_read_kernel_trace": (ctypes.c_int, [_P, _P, _P]),
    "dsa_set_stage_events": (ctypes.c_int, [_P, ctypes.c_int32]),
    "dsa_set_trace_buffer": (ctypes.c_int, [_P, ctypes.c_size_t]),
    "dsa_set_fault_injection": (ctypes.c_int, [ctypes.c_uint32, ctypes.c_uint32]),
    "dsa_indexer_scores": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, ctypes.c_int64, _P,
                                          ctypes.c_size_t, _P]),
    "dsa_topk": (ctypes.c_int, [_P, _P, _P, ctypes.c_int64, _P, _P, ctypes.c_size_t, _P]),
    "dsa_sparse_mla_fwd": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "dsa_sparse_mla_fwd_noalloc": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P]),
    "dsa_decode_step": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                       ctypes.c_size_t, _P]),
    "dsa_forward": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                   ctypes.c_size_t, _P]),
    "dsa_cache_append": (ctypes.c_int, [_P, _P, ctypes.c_int32, _P, _P, _P, _P, _P,
                                        ctypes.c_size_t, _P]),
    "dsa_indexer_kl": (ctypes.c_int, [_P, _P, ctypes.c_int64, _P, ctypes.c_int64, _P, ctypes.c_int64,
                                      _P, _P, ctypes.c_size_t, _P]),
    "dsa_indexer_backward": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, ctypes.c_int64, _P, _P, _P,
                                            _P, ctypes.c_size_t, _P]),
    "dsa_output_projection_ws_size": (ctypes.c_size_t, [_P, ctypes.c_int32]),
    "dsa_output_projection": (ctypes.c_int, [_P, ctypes.c_int32, _P, _P, _P, _P, _P, _P,
                                             ctypes.c_size_t, _P]),
}


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(f"libdsa.so not built at {path}: run long_context_sparse_04_b200.build")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = load()


class DSAError(RuntimeError):
    def __init__(self, name: str, status: int):
        self.status = status
        msg = LIB.dsa_last_error().decode()
        super().__init__(f"{name}: {LIB.dsa_status_string(status).decode()} {msg}")


def _ref(s):
    return ctypes.byref(s) if s is not None else None


def _call(name, *args, check=True):
    st = getattr(LIB, name)(*args)
    if check and st != DSA_OK:
        raise DSAError(name, st)
    return st


def dsa_workspace_size(dims, rows, op) -> int:
    return LIB.dsa_workspace_size(_ref(dims), _ref(rows), op)


def dsa_workspace_init(ws, ws_bytes, stream, check=True):
    return _call("dsa_workspace_init", ws, ws_bytes, stream, check=check)


def dsa_read_device_status(ws, stream):
    st, det = ctypes.c_int32(0), ctypes.c_int32(0)
    _call("dsa_read_device_status", ws, stream, ctypes.byref(st), ctypes.byref(det))
    return st.value, det.value


def dsa_read_kernel_trace(ws, stream) -> int:
    m = ctypes.c_uint32(0)
    _call("dsa_read_kernel_trace", ws, stream, ctypes.byref(m))
    return m.value


def dsa_set_stage_events(events):
    """events: list of 4 raw cudaEvent_t handles (ints), or [] to switch off."""
    arr = (ctypes.c_void_p * 4)(*[ctypes.c_void_p(e) for e in events]) if events else None
    return _call("dsa_set_stage_events", arr, len(events))


def dsa_set_trace_buffer(buf, nbytes):
    return _call("dsa_set_trace_buffer", buf, nbytes)


def dsa_set_fault_injection(spin_limit: int, faults: int, check=True):
    """Tests only: bounded-wait poll limit and DSA_FAULT_* bits of this thread's launches."""
    return _call("dsa_set_fault_injection", spin_limit, faults, check=check)


def dsa_indexer_scores(dims, rows, cache, q_idx, q_scale, w, scores, ld_scores, ws, ws_bytes,
                       stream, check=True):
    return _call("dsa_indexer_scores", _ref(dims), _ref(rows), _ref(cache), q_idx, q_scale, w,
                 scores, ld_scores, ws, ws_bytes, stream, check=check)


def dsa_topk(dims, rows, scores, ld_scores, idx, ws, ws_bytes, stream, check=True):
    return _call("dsa_topk", _ref(dims), _ref(rows), scores, ld_scores, idx, ws, ws_bytes,
                 stream, check=check)


def dsa_sparse_mla_fwd(dims, rows, cache, q, idx, out, lse, ws, ws_bytes, stream, check=True):
    return _call("dsa_sparse_mla_fwd", _ref(dims), _ref(rows), _ref(cache), q, idx, out, lse,
                 ws, ws_bytes, stream, check=check)


def dsa_sparse_mla_fwd_noalloc(dims, rows, cache, q, idx, out, lse, stream, check=True):
    return _call("dsa_sparse_mla_fwd_noalloc", _ref(dims), _ref(rows), _ref(cache), q, idx, out,
                 lse, stream, check=check)


def dsa_decode_step(dims, rows, cache, q_idx, q_scale, w, q, out, lse, dbg_scores, dbg_idx,
                    ws, ws_bytes, stream, check=True):
    return _call("dsa_decode_step", _ref(dims), _ref(rows), _ref(cache), q_idx, q_scale, w, q,
                 out, lse, dbg_scores, dbg_idx, ws, ws_bytes, stream, check=check)


def dsa_forward(dims, rows, cache, q_idx, q_scale, w, q, out, lse, idx_out, ws, ws_bytes,
                stream, check=True):
    return _call("dsa_forward", _ref(dims), _ref(rows), _ref(cache), q_idx, q_scale, w, q, out,
                 lse, idx_out, ws, ws_bytes, stream, check=check)


def dsa_cache_append(dims, cache, n_new, tok_seq, tok_pos, k_new, latent_new, ws, ws_bytes,
                     stream, check=True):
    return _call("dsa_cache_append", _ref(dims), _ref(cache), n_new, tok_seq, tok_pos, k_new,
                 latent_new, ws, ws_bytes, stream, check=check)


def dsa_output_projection_ws_size(dims, num_rows) -> int:
    return LIB.dsa_output_projection_ws_size(_ref(dims), num_rows)


def dsa_output_projection(dims, num_rows, o, w_uv, w_out, u, y, ws, ws_bytes, stream, check=True):
    return _call("dsa_output_projection", _ref(dims), num_rows, o, w_uv, w_out, u, y, ws, ws_bytes,
                 stream, check=check)


def dsa_indexer_kl(rows, scores, ld_scores, teacher, ld_teacher, grad, ld_grad, loss, ws, ws_bytes,
                   stream, check=True):
    return _call("dsa_indexer_kl", _ref(rows), scores, ld_scores, teacher, ld_teacher, grad, ld_grad,
                 loss, ws, ws_bytes, stream, check=check)


def dsa_indexer_backward(dims, rows, cache, q_idx, q_scale, w, grad, ld_grad, dq, dw, dk, ws, ws_bytes,
                         stream, check=True):
    return _call("dsa_indexer_backward", _ref(dims), _ref(rows), _ref(cache), q_idx, q_scale, w, grad,
                 ld_grad, dq, dw, dk, ws, ws_bytes, stream, check=check)
