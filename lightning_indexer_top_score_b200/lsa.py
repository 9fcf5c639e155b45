"""Thin ctypes binding of liblsa.so (include/lsa.h), same entry-point names.

Argument marshalling only: torch CUDA tensors are passed as raw device pointers together with
the current CUDA stream; every step of the computation runs in the library's kernels.  There is
no fallback of any kind -- if the library is missing or a tensor is not on a CUDA device, the call
raises.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblsa.so")

LSA_OK = 0
STATUS = {0: "LSA_OK", 1: "LSA_ERR_INVALID_ARG", 2: "LSA_ERR_UNSUPPORTED",
          3: "LSA_ERR_WORKSPACE", 4: "LSA_ERR_CUDA", 5: "LSA_ERR_DEVICE"}
DEVERR_QPOS, DEVERR_NONFINITE, DEVERR_INDEX, DEVERR_APPEND, DEVERR_INTERNAL = 1, 2, 4, 8, 16

EXPORTS = ("lsa_status_string", "lsa_version", "lsa_index_workspace_bytes", "lsa_index",
           "lsa_attend_workspace_bytes", "lsa_attend", "lsa_kv_append", "lsa_get_error",
           "lsa_index_noalloc", "lsa_launch_count", "lsa_quantize_fp8", "lsa_index_fp8", "lsa_attend_bwd",
           "lsa_kv_minmax", "lsa_index_minmax")
NOALLOC_SCRATCH_BYTES = 64 << 20

_lib = None


class LsaError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")
        self.status = status


def load(path: str = LIB_PATH):
    """Load liblsa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"liblsa.so not built at {path}; run "
                           "`python -m lightning_indexer_top_score_b200.build`")
    lib = ctypes.CDLL(path)
    P, i32, i64, sz, f32 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t,
                            ctypes.c_float)
    lib.lsa_status_string.restype = ctypes.c_char_p
    lib.lsa_status_string.argtypes = [i32]
    lib.lsa_version.restype = i32
    lib.lsa_launch_count.restype = ctypes.c_uint64
    lib.lsa_launch_count.argtypes = []
    lib.lsa_index_workspace_bytes.restype = sz
    lib.lsa_index_workspace_bytes.argtypes = [i32, i32, i32, i32, i64, i32, i32, i32, i32]
    lib.lsa_index.restype = i32
    lib.lsa_index.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i64, i32, i32, i32, i32, i32,
                              i32, P, P, P, P, sz, P]
    lib.lsa_attend_workspace_bytes.restype = sz
    lib.lsa_attend_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32, i32]
    lib.lsa_attend.restype = i32
    lib.lsa_attend.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i64, i32, i32, i32, f32,
                               P, P, P, sz, P]
    lib.lsa_kv_append.restype = i32
    lib.lsa_kv_append.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i64, i32, P, P]
    lib.lsa_get_error.restype = i32
    lib.lsa_get_error.argtypes = [P, P, P]
    lib.lsa_index_noalloc.restype = i32
    lib.lsa_index_noalloc.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i64, i32, i32, i32,
                                      i32, i32, i32, P, P, P]
    lib.lsa_quantize_fp8.restype = i32
    lib.lsa_quantize_fp8.argtypes = [P, i64, i64, i32, P, i64, P, i64, P, P]
    lib.lsa_attend_bwd.restype = i32
    lib.lsa_attend_bwd.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i64, i32, i32, i32, f32,
                                   P, P, P, P, P, P, P]
    lib.lsa_kv_minmax.restype = i32
    lib.lsa_kv_minmax.argtypes = [P, P, P, i32, i32, i32, i64, i32, P, P]
    lib.lsa_index_minmax.restype = i32
    lib.lsa_index_minmax.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i64, i32, i32, i32, i32,
                                     i32, i32, P, P, P, P, sz, P]
    lib.lsa_index_fp8.restype = i32
    lib.lsa_index_fp8.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i64, i32, i32, i32, P,
                                  P, P, sz, P]
    _lib = lib
    return lib


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("liblsa takes CUDA tensors only")
    if not t.is_contiguous():
        raise ValueError("liblsa takes contiguous tensors only")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, st):
    if st != LSA_OK:
        raise LsaError(fn, st)


def lsa_index_workspace_bytes(B, T, H_I, D_I, L_max, K_sparse, page=128, sub_block=8, M=0):
    return int(load().lsa_index_workspace_bytes(B, T, H_I, D_I, L_max, K_sparse, page, sub_block,
                                                M))


def lsa_attend_workspace_bytes(B, T, H, D_v, K_sparse, sink, swa):
    return int(load().lsa_attend_workspace_bytes(B, T, H, D_v, K_sparse, sink, swa))


def lsa_index(q_I, w_I, k_I, k_mean, kv_len, q_pos, K_sparse, sink, swa, page=128, sub_block=8,
              M=0, indices=None, scores_dbg=None, page_scores_dbg=None, ws=None, stream=None):
    """q_I [B,T,H_I,D_I] bf16, w_I [B,T,H_I] bf16, k_I [B,L_max,D_I] bf16, k_mean or None,
    kv_len [B] int32, q_pos [B,T] int32 -> indices [B,T,K_sparse] int32."""
    import torch
    B, T, H_I, D_I = q_I.shape
    L_max = k_I.shape[1]
    if indices is None:
        indices = torch.empty(B, T, K_sparse, dtype=torch.int32, device=q_I.device)
    need = lsa_index_workspace_bytes(B, T, H_I, D_I, L_max, K_sparse, page, sub_block, M)
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=q_I.device)
    st = load().lsa_index(_ptr(q_I), _ptr(w_I), _ptr(k_I), _ptr(k_mean), _ptr(kv_len),
                          _ptr(q_pos), B, T, H_I, D_I, L_max, K_sparse, sink, swa, page,
                          sub_block, M, _ptr(indices), _ptr(scores_dbg), _ptr(page_scores_dbg),
                          _ptr(ws), ws.numel(), _stream(stream))
    _check("lsa_index", st)
    return indices


def lsa_index_minmax(q_I, w_I, k_I, k_minmax, kv_len, q_pos, K_sparse, sink, swa, page=128,
                     sub_block=8, M=1024, indices=None, scores_dbg=None, page_scores_dbg=None,
                     ws=None, stream=None):
    """Hierarchical indexer whose stage 1 uses MinMax pooling: k_minmax [B, NB, 2*D_I] bf16 as
    lsa_kv_minmax writes it; other arguments as lsa_index (M >= 1)."""
    import torch
    B, T, H_I, D_I = q_I.shape
    L_max = k_I.shape[1]
    if indices is None:
        indices = torch.empty(B, T, K_sparse, dtype=torch.int32, device=q_I.device)
    need = lsa_index_workspace_bytes(B, T, H_I, D_I, L_max, K_sparse, page, sub_block, M)
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=q_I.device)
    st = load().lsa_index_minmax(_ptr(q_I), _ptr(w_I), _ptr(k_I), _ptr(k_minmax), _ptr(kv_len),
                                 _ptr(q_pos), B, T, H_I, D_I, L_max, K_sparse, sink, swa, page,
                                 sub_block, M, _ptr(indices), _ptr(scores_dbg),
                                 _ptr(page_scores_dbg), _ptr(ws), ws.numel(), _stream(stream))
    _check("lsa_index_minmax", st)
    return indices


def lsa_index_noalloc(q_I, w_I, k_I, k_mean, kv_len, q_pos, K_sparse, sink, swa, page=128,
                      sub_block=8, M=0, indices=None, device_error=None, stream=None):
    """lsa_index with no workspace argument, for callers that cannot allocate device memory: the
    library's own fixed scratch array (NOALLOC_SCRATCH_BYTES per GPU) is used instead.  The
    output buffer `indices` (and the optional int32 `device_error` word) are the caller's."""
    import torch
    B, T, H_I, D_I = q_I.shape
    L_max = k_I.shape[1]
    if indices is None:
        indices = torch.empty(B, T, K_sparse, dtype=torch.int32, device=q_I.device)
    st = load().lsa_index_noalloc(_ptr(q_I), _ptr(w_I), _ptr(k_I), _ptr(k_mean), _ptr(kv_len),
                                  _ptr(q_pos), B, T, H_I, D_I, L_max, K_sparse, sink, swa, page,
                                  sub_block, M, _ptr(indices), _ptr(device_error),
                                  _stream(stream))
    _check("lsa_index_noalloc", st)
    return indices


def _ptr_view(t):
    """Pointer of a CUDA tensor that may be a strided view (rows of a cache): its inner stride
    must be 1 and every stride positive; the callee is given the strides explicitly."""
    if not t.is_cuda:
        raise ValueError("liblsa takes CUDA tensors only")
    if t.dim() and (t.stride(-1) != 1 and t.dim() > 1 or any(st < 1 for st in t.stride())):
        raise ValueError(f"strided view {tuple(t.shape)} / {t.stride()} is not rows of elements")
    return ctypes.c_void_p(t.data_ptr())


def _row_stride(t, D):
    """Element stride between the rows of t viewed as [rows, D] (contiguous, or a 2-D view with
    unit inner stride, e.g. one token's slot of every sequence of a cache)."""
    if t.is_contiguous():
        return D
    if t.dim() == 2 and t.stride(1) == 1:
        return t.stride(0)
    raise ValueError(f"tensor of shape {tuple(t.shape)} / strides {t.stride()} is not rows of {D}")


def lsa_quantize_fp8(x, codes=None, scales=None, device_error=None, stream=None):
    """x bf16 [..., D] -> (codes uint8 [..., D], scales fp32 [...]): per-row E4M3 quantisation.
    codes / scales may be strided views (rows of a cache)."""
    import torch
    D = x.shape[-1]
    rows = x.numel() // D
    if codes is None:
        codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    s_stride = 1 if scales.is_contiguous() else scales.stride(0)
    if codes.numel() != x.numel() or scales.numel() != rows:
        raise ValueError("codes / scales do not match the rows of x")
    st = load().lsa_quantize_fp8(_ptr(x), _row_stride(x, D), rows, D, _ptr_view(codes),
                                 _row_stride(codes, D), _ptr_view(scales), s_stride,
                                 _ptr(device_error), _stream(stream))
    _check("lsa_quantize_fp8", st)
    return codes, scales


def lsa_index_fp8(q8, q_scale, w_I, k8, k_scale, kv_len, q_pos, K_sparse, sink, swa,
                  indices=None, scores_dbg=None, ws=None, stream=None):
    """Flat indexer on FP8 codes: q8 uint8 [B,T,H_I,128] + q_scale [B,T,H_I], w_I bf16 [B,T,H_I],
    k8 uint8 [B,L_max,128] + k_scale [B,L_max] -> indices [B,T,K_sparse] int32."""
    import torch
    B, T, H_I, D_I = q8.shape
    L_max = k8.shape[1]
    if indices is None:
        indices = torch.empty(B, T, K_sparse, dtype=torch.int32, device=q8.device)
    need = lsa_index_workspace_bytes(B, T, H_I, D_I, L_max, K_sparse, 128, 8, 0)
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=q8.device)
    st = load().lsa_index_fp8(_ptr(q8), _ptr(q_scale), _ptr(w_I), _ptr(k8), _ptr(k_scale),
                              _ptr(kv_len), _ptr(q_pos), B, T, H_I, D_I, L_max, K_sparse, sink,
                              swa, _ptr(indices), _ptr(scores_dbg), _ptr(ws), ws.numel(),
                              _stream(stream))
    _check("lsa_index_fp8", st)
    return indices


def lsa_attend(q, c_kv, indices, kv_len, q_pos, sink, swa, scale, out=None, lse=None, ws=None,
               stream=None):
    """q [B,T,H,576] bf16, c_kv [B,L_max,576] bf16, indices [B,T,K] int32 -> (out [B,T,H,512]
    bf16, lse [B,T,H] fp32)."""
    import torch
    B, T, H, Dqk = q.shape
    L_max = c_kv.shape[1]
    K = indices.shape[-1] if indices is not None else 0
    if out is None:
        out = torch.empty(B, T, H, 512, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(B, T, H, dtype=torch.float32, device=q.device)
    need = lsa_attend_workspace_bytes(B, T, H, 512, K, sink, swa)
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    st = load().lsa_attend(_ptr(q), _ptr(c_kv), _ptr(indices), _ptr(kv_len), _ptr(q_pos), B, T,
                           H, Dqk, 512, L_max, K, sink, swa, float(scale), _ptr(out), _ptr(lse),
                           _ptr(ws), ws.numel(), _stream(stream))
    _check("lsa_attend", st)
    return out, lse


def lsa_attend_bwd(q, c_kv, indices, kv_len, q_pos, sink, swa, scale, dout, out=None, lse=None,
                   dq=None, dc_kv=None, device_error=None, stream=None):
    """Backward of lsa_attend: dout [B,T,H,512] bf16 -> (dq [B,T,H,576] fp32, dc_kv [B,L_max,576]
    fp32).  out / lse: the forward's outputs (both or neither; without them lse and D are
    recomputed).  dc_kv, if given, is accumulated into (zero it first); otherwise a zeroed one
    is made."""
    import torch
    B, T, H, Dqk = q.shape
    L_max = c_kv.shape[1]
    K = indices.shape[-1] if indices is not None else 0
    if dq is None:
        dq = torch.empty(B, T, H, Dqk, dtype=torch.float32, device=q.device)
    if dc_kv is None:
        dc_kv = torch.zeros(B, L_max, Dqk, dtype=torch.float32, device=q.device)
    st = load().lsa_attend_bwd(_ptr(q), _ptr(c_kv), _ptr(indices), _ptr(kv_len), _ptr(q_pos), B,
                               T, H, Dqk, 512, L_max, K, sink, swa, float(scale), _ptr(out),
                               _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dc_kv), _ptr(device_error),
                               _stream(stream))
    _check("lsa_attend_bwd", st)
    return dq, dc_kv


def lsa_kv_append(kv_len_old, k_I_new=None, k_I=None, k_mean=None, c_new=None, c_kv=None,
                  sub_block=8, device_error=None, stream=None):
    """Append n_new tokens per sequence at kv_len_old[b]; refresh the sub-block means."""
    src = k_I_new if k_I_new is not None else c_new
    B, n_new = src.shape[0], src.shape[1]
    L_max = (k_I if k_I is not None else c_kv).shape[1]
    D_I = k_I_new.shape[-1] if k_I_new is not None else 0
    D_qk = c_new.shape[-1] if c_new is not None else 0
    st = load().lsa_kv_append(_ptr(k_I_new), _ptr(k_I), _ptr(k_mean), _ptr(c_new), _ptr(c_kv),
                              _ptr(kv_len_old), B, n_new, D_I, D_qk, L_max, sub_block,
                              _ptr(device_error), _stream(stream))
    _check("lsa_kv_append", st)


def lsa_kv_minmax(kv_len_old, n_new, k_I, k_minmax, sub_block=8, device_error=None,
                  stream=None):
    """Refresh the MinMax rows of the sub-blocks touched by n_new tokens appended at
    kv_len_old[b] (their keys already in k_I)."""
    B, L_max, D_I = k_I.shape
    st = load().lsa_kv_minmax(_ptr(k_I), _ptr(k_minmax), _ptr(kv_len_old), B, int(n_new), D_I,
                              L_max, sub_block, _ptr(device_error), _stream(stream))
    _check("lsa_kv_minmax", st)


def lsa_launch_count() -> int:
    """Kernels the library has launched since it was loaded (host-side count at launch)."""
    return int(load().lsa_launch_count())


def lsa_get_error(ws, stream=None) -> int:
    """Synchronise the stream and return the device error word of the last call on ws."""
    code = ctypes.c_int32(0)
    st = load().lsa_get_error(_ptr(ws), ctypes.byref(code), _stream(stream))
    if st not in (LSA_OK, 5):
        raise LsaError("lsa_get_error", st)
    return int(code.value)
