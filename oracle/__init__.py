"""fp64 CPU oracle for the LSA layer hot path (LongCat Sparse Attention, arXiv 2608.01662).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` are the only callers.  The product path never imports this package, and this
package imports nothing from the product package.

The arithmetic lives in ``lsa_oracle.c`` (plain C, fp64, OpenMP over independent query rows);
this module only builds it with gcc and marshals numpy arrays through ctypes.  bf16 tensors are
passed as ``uint16`` arrays holding the raw bf16 bit patterns.

Parity pins: every function here is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py`` against closed forms, library routines (numpy matmul, a textbook
causal softmax attention in torch float64), brute-force ranking and hand-derived fixtures under
``tests/golden/``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lsa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liblsa_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile lsa_oracle.c into liblsa_oracle.so next to it (gcc, -O2, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
           "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.orc_num_threads.restype = i32
    lib.orc_set_num_threads.argtypes = [i32]
    lib.orc_regions.argtypes = [i64, i32, i32, P]
    lib.orc_score_one.argtypes = [P, P, P, i32, i32]
    lib.orc_score_one.restype = f64
    lib.orc_scores.argtypes = [P, P, P, i32, i32, P, i64, P]
    lib.orc_topk.argtypes = [P, P, i64, i32, P]
    lib.orc_topk.restype = i64
    lib.orc_block_means.argtypes = [P, i64, i32, i32, P]
    lib.orc_page_score.argtypes = [P, P, P, i32, i32, i64, i32, i32, i64]
    lib.orc_page_score.restype = f64
    lib.orc_index_query.argtypes = [P, P, P, P, i32, i32, i64, i64, i32, i32, i32, i32, i32, i32, P]
    lib.orc_index_query.restype = i64
    lib.orc_index.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i64, i32, i32, i32, i32, i32,
                              i32, P]
    lib.orc_block_minmax.argtypes = [P, i64, i32, i32, P]
    lib.orc_page_score_minmax.argtypes = [P, P, P, i32, i32, i64, i32, i32, i64]
    lib.orc_page_score_minmax.restype = f64
    lib.orc_index_query_pool.argtypes = [P, P, P, P, i32, i32, i32, i64, i64, i32, i32, i32, i32,
                                         i32, i32, P]
    lib.orc_index_query_pool.restype = i64
    lib.orc_index_pool.argtypes = [P, P, P, P, i32, P, P, i32, i32, i32, i32, i64, i32, i32, i32,
                                   i32, i32, i32, P]
    lib.orc_select_query.argtypes = [P, P, i64, i32, i32, i32, i32, i32, P]
    lib.orc_select_query.restype = i64
    lib.orc_attend_query.argtypes = [P, P, P, i32, i64, i32, i32, i32, i32, i32, f64, P, P]
    lib.orc_attend_query_branches.argtypes = [P, P, P, i32, i64, i32, i32, i32, i32, i32, f64, P,
                                              P]
    lib.orc_attend.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, i64, i32, i32, i32, f64, P, P]
    lib.orc_attend_bwd_query.argtypes = [P, P, P, i32, i64, i32, i32, i32, i32, i32, f64, P, P, P]
    lib.orc_attend_bwd.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, i64, i32, i32, i32, f64,
                                   P, P, P]
    lib.orc_e4m3_value.argtypes = [ctypes.c_uint8]
    lib.orc_e4m3_value.restype = f64
    lib.orc_e4m3_encode.argtypes = [ctypes.c_float]
    lib.orc_e4m3_encode.restype = ctypes.c_uint8
    lib.orc_quantize_e4m3.argtypes = [P, i64, i32, P, P]
    lib.orc_score_one_fp8.argtypes = [P, P, P, P, ctypes.c_float, i32, i32]
    lib.orc_score_one_fp8.restype = f64
    lib.orc_scores_fp8.argtypes = [P, P, P, P, P, i32, i32, P, i64, P]
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"bf16 tensors are passed as uint16 bit patterns, got {a.dtype}")
    return a


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int32)


def num_threads() -> int:
    return int(_load().orc_num_threads())


def set_num_threads(n: int) -> None:
    _load().orc_set_num_threads(int(n))


def regions(t: int, sink: int, swa: int):
    """Streaming-aware region split of query t: ((sink_lo, sink_hi), (swa_lo, swa_hi),
    (dyn_lo, dyn_hi)), half-open ranges."""
    r = np.zeros(6, dtype=np.int64)
    _load().orc_regions(int(t), int(sink), int(swa), _ptr(r))
    return (int(r[0]), int(r[1])), (int(r[2]), int(r[3])), (int(r[4]), int(r[5]))


def score_one(q, w, key) -> float:
    """Eq. 1 for one (query, key): q [H, D], w [H], key [D] (bf16 bits)."""
    q, w, key = _u16(q), _u16(w), _u16(key)
    H, D = q.shape
    return float(_load().orc_score_one(_ptr(q), _ptr(w), _ptr(key), H, D))


def scores(q, w, k_seq, pos) -> np.ndarray:
    """Eq. 1 of one query against k_seq[pos] (k_seq [L, D])."""
    q, w, k_seq = _u16(q), _u16(w), _u16(k_seq)
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    H, D = q.shape
    out = np.zeros(len(pos), dtype=np.float64)
    _load().orc_scores(_ptr(q), _ptr(w), _ptr(k_seq), H, D, _ptr(pos), len(pos), _ptr(out))
    return out


def attend_bwd_query(q, c_seq, idx, t: int, sink: int, swa: int, Dv: int, scale: float, dout,
                     dc_seq=None):
    """Backward of one query row's attention: q [H, Dqk] (bf16 bits), c_seq [L, Dqk] (bf16 bits),
    dout [H, Dv] (float) -> (dq [H, Dqk] fp64, dc_seq [L, Dqk] fp64 with this row's gradients
    of its S_t rows added)."""
    q, c_seq = _u16(q), _u16(c_seq)
    idx = _i32(idx)
    dout = np.ascontiguousarray(dout, dtype=np.float64)
    H, Dqk = q.shape
    if dc_seq is None:
        dc_seq = np.zeros((c_seq.shape[0], Dqk), dtype=np.float64)
    dq = np.zeros((H, Dqk), dtype=np.float64)
    _load().orc_attend_bwd_query(_ptr(q), _ptr(c_seq), _ptr(idx), len(idx), int(t), int(sink),
                                 int(swa), H, Dqk, int(Dv), float(scale), _ptr(dout), _ptr(dq),
                                 _ptr(dc_seq))
    return dq, dc_seq


def attend_bwd(q, c, idx, q_pos, sink: int, swa: int, Dv: int, scale: float, dout):
    """Batched backward: q [B,T,H,Dqk], c [B,Lmax,Dqk] (bf16 bits), idx [B,T,K], q_pos [B,T],
    dout [B,T,H,Dv] -> (dq [B,T,H,Dqk], dc [B,Lmax,Dqk]) fp64."""
    q, c = _u16(q), _u16(c)
    idx, q_pos = _i32(idx), _i32(q_pos)
    dout = np.ascontiguousarray(dout, dtype=np.float64)
    B, T, H, Dqk = q.shape
    Lmax = c.shape[1]
    dq = np.zeros((B, T, H, Dqk), dtype=np.float64)
    dc = np.zeros((B, Lmax, Dqk), dtype=np.float64)
    _load().orc_attend_bwd(_ptr(q), _ptr(c), _ptr(idx), _ptr(q_pos), B, T, H, Dqk, int(Dv), Lmax,
                           idx.shape[-1], int(sink), int(swa), float(scale), _ptr(dout), _ptr(dq),
                           _ptr(dc))
    return dq, dc


def e4m3_value(code: int) -> float:
    """Value of one E4M3 code (OCP 8-bit floating point: bias 7, 3 mantissa bits, max 448)."""
    return float(_load().orc_e4m3_value(int(code) & 0xFF))


def e4m3_encode(y: float) -> int:
    """Nearest E4M3 code to the fp32 value y (ties to even, saturating at 448)."""
    return int(_load().orc_e4m3_encode(float(y)))


def quantize_e4m3(x):
    """Per-row FP8 quantisation of bf16 rows x [..., D]: (codes uint8 [..., D], scales fp32
    [...]) with scale = amax / 448 and code = E4M3(x / scale), both quotients in fp32."""
    x = _u16(x)
    D = x.shape[-1]
    rows = x.size // D
    codes = np.zeros(x.shape, dtype=np.uint8)
    scales = np.zeros(x.shape[:-1], dtype=np.float32)
    _load().orc_quantize_e4m3(_ptr(x), rows, D, _ptr(codes), _ptr(scales))
    return codes, scales


def score_one_fp8(q8, qs, w, k8, ks) -> float:
    """Eq. 1 on decoded FP8 rows: q8 [H, D] codes, qs [H] fp32, w [H] bf16 bits, key k8 [D], ks."""
    q8 = np.ascontiguousarray(q8, dtype=np.uint8)
    qs = np.ascontiguousarray(qs, dtype=np.float32)
    w = _u16(w)
    k8 = np.ascontiguousarray(k8, dtype=np.uint8)
    H, D = q8.shape
    return float(_load().orc_score_one_fp8(_ptr(q8), _ptr(qs), _ptr(w), _ptr(k8), float(ks), H, D))


def scores_fp8(q8, qs, w, k8_seq, ks_seq, pos) -> np.ndarray:
    """FP8 Eq. 1 of one query against keys k8_seq[pos] (k8_seq [L, D] codes, ks_seq [L])."""
    q8 = np.ascontiguousarray(q8, dtype=np.uint8)
    qs = np.ascontiguousarray(qs, dtype=np.float32)
    w = _u16(w)
    k8_seq = np.ascontiguousarray(k8_seq, dtype=np.uint8)
    ks_seq = np.ascontiguousarray(ks_seq, dtype=np.float32)
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    H, D = q8.shape
    out = np.zeros(len(pos), dtype=np.float64)
    _load().orc_scores_fp8(_ptr(q8), _ptr(qs), _ptr(w), _ptr(k8_seq), _ptr(ks_seq), H, D,
                           _ptr(pos), len(pos), _ptr(out))
    return out


def topk(score, pos, K: int):
    """arg-top-K by (score desc, pos asc); returns (indices [K] int32 ascending, -1 padded, m)."""
    score = np.ascontiguousarray(score, dtype=np.float64)
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    out = np.zeros(K, dtype=np.int32)
    m = _load().orc_topk(_ptr(score), _ptr(pos), len(score), int(K), _ptr(out))
    return out, int(m)


def block_means(k_seq, L: int, B: int) -> np.ndarray:
    """Sub-block means (fp64) of k_seq[0:L] with block size B -> [ceil(L/B), D]."""
    k_seq = _u16(k_seq)
    D = k_seq.shape[1]
    nb = (L + B - 1) // B
    out = np.zeros((nb, D), dtype=np.float64)
    _load().orc_block_means(_ptr(k_seq), int(L), D, int(B), _ptr(out))
    return out


def page_score(q, w, kmean_seq, L: int, P: int, B: int, p: int) -> float:
    """Eq. 9 of one query for page p from the stored bf16 means kmean_seq [NB, D]."""
    q, w, kmean_seq = _u16(q), _u16(w), _u16(kmean_seq)
    H, D = q.shape
    return float(_load().orc_page_score(_ptr(q), _ptr(w), _ptr(kmean_seq), H, D, int(L), int(P),
                                        int(B), int(p)))


POOLING = {"mean": 0, "minmax": 1}


def index_query(q, w, k_seq, kmean_seq, L, t, K, sink, swa, page=128, sub_block=8, M=0,
                pooling="mean"):
    """Full LSA indexer for one query (flat when M == 0, hierarchical when M > 0).  With
    pooling='minmax', kmean_seq holds the (k_max, k_min) rows [NB, 2D] instead of the means."""
    q, w, k_seq = _u16(q), _u16(w), _u16(k_seq)
    km = _u16(kmean_seq) if kmean_seq is not None else None
    H, D = q.shape
    out = np.zeros(K, dtype=np.int32)
    m = _load().orc_index_query_pool(_ptr(q), _ptr(w), _ptr(k_seq),
                                     _ptr(km) if km is not None else None, POOLING[pooling], H, D,
                                     int(L), int(t), int(K), int(sink), int(swa), int(page),
                                     int(sub_block), int(M), _ptr(out))
    return out, int(m)


def index(q, w, k, kmean, kv_len, q_pos, K, sink, swa, page=128, sub_block=8, M=0,
          pooling="mean"):
    """Batched indexer: q [B,T,H,D], w [B,T,H], k [B,Lmax,D], kmean [B,NBmax,D] (pooling
    'mean') or [B,NBmax,2D] (pooling 'minmax') or None, kv_len [B], q_pos [B,T]
    -> indices [B,T,K] int32."""
    q, w, k = _u16(q), _u16(w), _u16(k)
    km = _u16(kmean) if kmean is not None else None
    kv_len, q_pos = _i32(kv_len), _i32(q_pos)
    Bn, T, H, D = q.shape
    Lmax = k.shape[1]
    out = np.zeros((Bn, T, K), dtype=np.int32)
    _load().orc_index_pool(_ptr(q), _ptr(w), _ptr(k), _ptr(km) if km is not None else None,
                           POOLING[pooling], _ptr(kv_len), _ptr(q_pos), Bn, T, H, D, Lmax, int(K),
                           int(sink), int(swa), int(page), int(sub_block), int(M), _ptr(out))
    return out


def block_minmax(k_seq, L: int, B: int) -> np.ndarray:
    """MinMax pooling rows (Sec. 5.3.5) of k_seq[0:L] with sub-block size B -> [ceil(L/B), 2D]
    fp64, row n = (element-wise max, element-wise min) over the sub-block's tokens."""
    k_seq = _u16(k_seq)
    D = k_seq.shape[1]
    nb = (L + B - 1) // B
    out = np.zeros((nb, 2 * D), dtype=np.float64)
    _load().orc_block_minmax(_ptr(k_seq), int(L), D, int(B), _ptr(out))
    return out


def page_score_minmax(q, w, kmm_seq, L: int, P: int, B: int, p: int) -> float:
    """Page score with MinMax pooling (Sec. 5.3.5's sub-block term in place of q . k_mean in
    Eq. 9) of one query for page p from the stored bf16 rows kmm_seq [NB, 2D]."""
    q, w, kmm_seq = _u16(q), _u16(w), _u16(kmm_seq)
    H, D = q.shape
    return float(_load().orc_page_score_minmax(_ptr(q), _ptr(w), _ptr(kmm_seq), H, D, int(L),
                                               int(P), int(B), int(p)))


def select_query(tok_scores, page_scores, t, K, sink, swa, page=128, M=0):
    """Selection steps only, on externally computed fp32 scores: tok_scores indexed by absolute
    position, page_scores by absolute page id (unused when M == 0)."""
    ts = np.ascontiguousarray(tok_scores, dtype=np.float32)
    ps = np.ascontiguousarray(page_scores if page_scores is not None else np.zeros(1),
                              dtype=np.float32)
    out = np.zeros(K, dtype=np.int32)
    m = _load().orc_select_query(_ptr(ts), _ptr(ps), int(t), int(K), int(sink), int(swa),
                                 int(page), int(M), _ptr(out))
    return out, int(m)


def attend_query(q, c_seq, idx, t, sink, swa, Dv, scale, branches=False):
    """Attention of one query: q [H, Dqk], c_seq [Lmax, Dqk], idx [K] -> (out [H, Dv], lse [H]).
    branches=True computes the contiguous and sparse branches apart and merges them by LSE."""
    q, c_seq = _u16(q), _u16(c_seq)
    idx = _i32(idx)
    H, Dqk = q.shape
    out = np.zeros((H, Dv), dtype=np.float64)
    lse = np.zeros(H, dtype=np.float64)
    fn = _load().orc_attend_query_branches if branches else _load().orc_attend_query
    fn(_ptr(q), _ptr(c_seq), _ptr(idx), len(idx), int(t), int(sink), int(swa), H, Dqk, int(Dv),
       float(scale), _ptr(out), _ptr(lse))
    return out, lse


def attend(q, c, idx, q_pos, sink, swa, Dv, scale):
    """Batched attention: q [B,T,H,Dqk], c [B,Lmax,Dqk], idx [B,T,K], q_pos [B,T]
    -> (out [B,T,H,Dv] fp64, lse [B,T,H] fp64)."""
    q, c = _u16(q), _u16(c)
    idx, q_pos = _i32(idx), _i32(q_pos)
    Bn, T, H, Dqk = q.shape
    Lmax = c.shape[1]
    K = idx.shape[-1]
    out = np.zeros((Bn, T, H, Dv), dtype=np.float64)
    lse = np.zeros((Bn, T, H), dtype=np.float64)
    _load().orc_attend(_ptr(q), _ptr(c), _ptr(idx), _ptr(q_pos), Bn, T, H, Dqk, int(Dv), Lmax,
                       K, int(sink), int(swa), float(scale), _ptr(out), _ptr(lse))
    return out, lse
