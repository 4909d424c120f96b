"""ctypes front end of the CPU oracle (oracle.c).

TEST INFRASTRUCTURE ONLY: tests/, __graft_entry__.smoke() and the CPU-baseline
leg of bench.py may import this module; the product path never does.  Every
function takes and returns numpy arrays; the arithmetic lives in oracle.c and
is documented there with the passages it follows.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        c_f, c_d, c_i, c_p = ctypes.c_float, ctypes.c_double, ctypes.c_int, ctypes.c_void_p
        L.oracle_e4m3_value.restype = c_d
        L.oracle_e4m3_value.argtypes = [ctypes.c_uint]
        L.oracle_e4m3_from_f32.restype = ctypes.c_uint
        L.oracle_e4m3_from_f32.argtypes = [c_f]
        L.oracle_fwht64.restype = None
        L.oracle_fwht64.argtypes = [c_p]
        L.oracle_fwht128.restype = None
        L.oracle_fwht128.argtypes = [c_p]
        L.oracle_quantize.restype = c_i
        L.oracle_quantize.argtypes = [c_p, c_i, c_i, c_i, c_i, c_i, c_p, c_p]
        L.oracle_attention_rows.restype = c_i
        L.oracle_attention_rows.argtypes = [c_p, c_p, c_p, c_i, c_i, c_i, c_i, c_i, c_i, c_d,
                                            c_p, c_i, c_p]
        L.oracle_leanp_slope.restype = c_f
        L.oracle_leanp_slope.argtypes = [c_f, c_f, c_i]
        L.oracle_leanp_block_shift.restype = c_i
        L.oracle_leanp_block_shift.argtypes = [c_f, c_f, c_f]
        L.oracle_leanp_code.restype = ctypes.c_uint
        L.oracle_leanp_code.argtypes = [c_f, c_f, c_f, c_i, c_i]
        L.oracle_leanp_batch.restype = None
        L.oracle_leanp_batch.argtypes = [c_p, c_p, c_p, c_p, c_p, c_i, c_p, c_p]
        L.oracle_fp8_model_rows.restype = c_i
        L.oracle_fp8_model_rows.argtypes = [c_p, c_p, c_p, c_p, c_p, c_p, c_i, c_i, c_i, c_i,
                                            c_i, c_i, c_i, c_f, c_i, c_p, c_i, c_p, c_p]
        L.oracle_attention_lse_rows.restype = c_i
        L.oracle_attention_lse_rows.argtypes = [c_p, c_p, c_i, c_i, c_i, c_i, c_i, c_d, c_p, c_i, c_p]
        L.oracle_exactp_code.restype = ctypes.c_uint
        L.oracle_exactp_code.argtypes = [c_f, c_f, c_f, c_i, c_i]
        L.oracle_num_threads.restype = c_i
        L.oracle_num_threads.argtypes = []
        _lib = L
    return _lib


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return lib().oracle_num_threads()


# --- e4m3 codec --------------------------------------------------------------

def e4m3_value(code: int) -> float:
    return lib().oracle_e4m3_value(int(code))


def e4m3_values() -> np.ndarray:
    """Decoded value of every code 0..255 (fp64; NaN for 0x7F and 0xFF)."""
    return np.array([lib().oracle_e4m3_value(c) for c in range(256)], dtype=np.float64)


def e4m3_from_f32(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float32).reshape(-1)
    return np.array([lib().oracle_e4m3_from_f32(float(v)) for v in x], dtype=np.uint8)


def dequantize(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """codes [B,S,H,D] uint8, scale [B,H] -> fp64 values value(code) * scale."""
    table = e4m3_values()
    vals = table[codes]
    B, S, H, D = codes.shape
    return vals * np.asarray(scale, dtype=np.float64).reshape(B, 1, H, 1)


# --- Hadamard and quantizer --------------------------------------------------

def fwht64(x) -> np.ndarray:
    """Orthonormal 64-point transform of each row of x [..., 64] (fp32 steps)."""
    x = _c(x, np.float32).copy()
    flat = x.reshape(-1, 64)
    for r in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[r])
        lib().oracle_fwht64(_ptr(row))
        flat[r] = row
    return flat.reshape(x.shape)


def fwht128(x) -> np.ndarray:
    """Orthonormal 128-point transform of each row of x [..., 128] (fp32 steps)."""
    x = _c(x, np.float32).copy()
    flat = x.reshape(-1, 128)
    for r in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[r])
        lib().oracle_fwht128(_ptr(row))
        flat[r] = row
    return flat.reshape(x.shape)


def quantize(x, hadamard: bool = False):
    """x [B,S,H,D] (fp32, or bf16 widened to fp32) -> (codes uint8 [B,S,H,D], scale fp32 [B,H])."""
    x = _c(x, np.float32)
    B, S, H, D = x.shape
    codes = np.empty(x.shape, dtype=np.uint8)
    scale = np.empty((B, H), dtype=np.float32)
    rc = lib().oracle_quantize(_ptr(x), B, S, H, D, int(bool(hadamard)), _ptr(codes), _ptr(scale))
    if rc != 0:
        raise ValueError("oracle_quantize: bad arguments")
    return codes, scale


# --- attention ---------------------------------------------------------------

def attention(q, k, v, sm_scale=None, rows=None) -> np.ndarray:
    """Causal attention in fp64.  q [B,S,Hq,Dqk], k [B,S,Hkv,Dqk], v [B,S,Hkv,Dv].
    Returns o [B,S,Hq,Dv], or [B,len(rows),Hq,Dv] for the listed query rows."""
    q = _c(q, np.float64); k = _c(k, np.float64); v = _c(v, np.float64)
    B, S, Hq, Dqk = q.shape
    Hkv, Dv = k.shape[2], v.shape[3]
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(Dqk)
    r = None if rows is None else _c(rows, np.int32)
    n = S if rows is None else len(r)
    o = np.empty((B, n, Hq, Dv), dtype=np.float64)
    rc = lib().oracle_attention_rows(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, S, Dqk, Dv,
                                     float(sm_scale), _ptr(r), n, _ptr(o))
    if rc != 0:
        raise ValueError("oracle_attention_rows: bad arguments")
    return o


def attention_lse(q, k, sm_scale=None, rows=None) -> np.ndarray:
    """Log-sum-exp of each row's causal scores in fp64: lse [B, Hq, S or len(rows)]."""
    q = _c(q, np.float64); k = _c(k, np.float64)
    B, S, Hq, Dqk = q.shape
    Hkv = k.shape[2]
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(Dqk)
    r = None if rows is None else _c(rows, np.int32)
    n = S if rows is None else len(r)
    lse = np.empty((B, Hq, n), dtype=np.float64)
    rc = lib().oracle_attention_lse_rows(_ptr(q), _ptr(k), B, Hq, Hkv, S, Dqk, float(sm_scale), _ptr(r), n,
                                         _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attention_lse_rows: bad arguments")
    return lse


# --- Lean P ------------------------------------------------------------------

def leanp_slope(q_s: float, k_s: float, dqk: int) -> np.float32:
    return np.float32(lib().oracle_leanp_slope(float(q_s), float(k_s), int(dqk)))


def leanp_block_shift(m, bmax, A) -> int:
    return lib().oracle_leanp_block_shift(float(m), float(bmax), float(A))


def leanp_code(s, m, A, j, masked=False) -> int:
    return lib().oracle_leanp_code(float(s), float(m), float(A), int(j), int(bool(masked)))


def exactp_code(s, m, A, j, masked=False) -> int:
    """The exact-P ablation's code: e4m3 of fl32(exp2((s - m) A / 8 + j))."""
    return lib().oracle_exactp_code(float(s), float(m), float(A), int(j), int(bool(masked)))


def leanp_batch(s, m, bmax, A, masked=None):
    """Element-wise Lean-P codes and block shifts (fp32 inputs, same length)."""
    s = _c(s, np.float32); m = _c(m, np.float32); bmax = _c(bmax, np.float32); A = _c(A, np.float32)
    n = s.size
    mk = None if masked is None else _c(masked, np.uint8)
    code = np.empty(n, dtype=np.uint8)
    j = np.empty(n, dtype=np.int32)
    lib().oracle_leanp_batch(_ptr(s), _ptr(m), _ptr(bmax), _ptr(A), _ptr(mk), n, _ptr(code), _ptr(j))
    return code, j


def fp8_model(qc, kc, vc, q_s, k_s, v_s, exact_p=False, rows=None, rescale_log2=0.0, p_mode=None,
              return_lse=False, kv_tile=128):
    """The FP8 pipeline replayed on the CPU (see oracle.c).  Codes uint8 BSHD,
    scales fp32 [B,H].  rescale_log2 = 0: exact running max; > 0: the reference
    max moves only when a tile max exceeds it by more than that many binades.
    kv_tile: keys per KV tile (128 or 256), the unit at which that decision
    is taken.
    p_mode: 0 Lean-P codes (default), 1 exact fp64 weights (exact_p=True),
    2 exact exp2 rounded to e4m3 (the exact-P ablation).
    Returns o fp64 [B, S or len(rows), Hq, Dv] (and lse [B, Hq, rows] with
    return_lse: ln 2 (m A/8 + log2 l) from the replay's own row sum)."""
    if p_mode is None:
        p_mode = 1 if exact_p else 0
    qc = _c(qc, np.uint8); kc = _c(kc, np.uint8); vc = _c(vc, np.uint8)
    q_s = _c(q_s, np.float32); k_s = _c(k_s, np.float32); v_s = _c(v_s, np.float32)
    B, S, Hq, Dqk = qc.shape
    Hkv, Dv = kc.shape[2], vc.shape[3]
    r = None if rows is None else _c(rows, np.int32)
    n = S if rows is None else len(r)
    o = np.empty((B, n, Hq, Dv), dtype=np.float64)
    lse = np.empty((B, Hq, n), dtype=np.float64) if return_lse else None
    rc = lib().oracle_fp8_model_rows(_ptr(qc), _ptr(kc), _ptr(vc), _ptr(q_s), _ptr(k_s), _ptr(v_s),
                                     B, Hq, Hkv, S, Dqk, Dv, int(p_mode), ctypes.c_float(rescale_log2), int(kv_tile),
                                     _ptr(r), n, _ptr(o),
                                     _ptr(lse))
    if rc == -2:
        raise ArithmeticError("oracle_fp8_model_rows: a block shift fell below its bound (reference max too stale)")
    if rc != 0:
        raise ValueError("oracle_fp8_model_rows: bad arguments")
    return (o, lse) if return_lse else o


# --- variable-length (packed) batches ------------------------------------------
# A packed batch holds independent sequences back to back: sequence s is rows
# cu[s] .. cu[s+1]-1 of every [T, H, D] tensor.  Each function below is its
# fixed-length counterpart applied to every sequence alone (a batch of one),
# results placed at the sequence's rows; nothing else is computed.

def _spans(cu):
    cu = [int(x) for x in cu]
    return [(cu[s], cu[s + 1]) for s in range(len(cu) - 1)]


def attention_varlen(q, k, v, cu, sm_scale=None) -> np.ndarray:
    """q [T,Hq,Dqk], k [T,Hkv,Dqk], v [T,Hkv,Dv] -> o [T,Hq,Dv] fp64, causal per sequence."""
    T, Hq = q.shape[0], q.shape[1]
    o = np.zeros((T, Hq, v.shape[2]), dtype=np.float64)
    for r0, r1 in _spans(cu):
        if r1 > r0:
            o[r0:r1] = attention(q[None, r0:r1], k[None, r0:r1], v[None, r0:r1], sm_scale=sm_scale)[0]
    return o


def attention_lse_varlen(q, k, cu, sm_scale=None) -> np.ndarray:
    """Log-sum-exp of each row's causal scores within its sequence: lse [Hq, T] fp64."""
    T, Hq = q.shape[0], q.shape[1]
    lse = np.zeros((Hq, T), dtype=np.float64)
    for r0, r1 in _spans(cu):
        if r1 > r0:
            lse[:, r0:r1] = attention_lse(q[None, r0:r1], k[None, r0:r1], sm_scale=sm_scale)[0]
    return lse


def quantize_varlen(x, cu, hadamard: bool = False):
    """x [T,H,D] -> (codes uint8 [T,H,D], scale fp32 [nseq,H]): each sequence quantized alone; an
    empty sequence gets the scale of an all-zero input."""
    x = _c(x, np.float32)
    T, H, D = x.shape
    spans = _spans(cu)
    codes = np.zeros((T, H, D), dtype=np.uint8)
    scale = np.empty((len(spans), H), dtype=np.float32)
    for s, (r0, r1) in enumerate(spans):
        part = x[None, r0:r1] if r1 > r0 else np.zeros((1, 1, H, D), dtype=np.float32)
        c, sc = quantize(part, hadamard=hadamard)
        if r1 > r0:
            codes[r0:r1] = c[0]
        scale[s] = sc[0]
    return codes, scale


def fp8_model_varlen(qc, kc, vc, q_s, k_s, v_s, cu, rescale_log2=0.0, p_mode=0, return_lse=False, kv_tile=128):
    """fp8_model over a packed batch: codes [T,H,D], scales [nseq,H].  Returns o [T,Hq,Dv] (and
    lse [Hq,T] with return_lse)."""
    T, Hq = qc.shape[0], qc.shape[1]
    o = np.zeros((T, Hq, vc.shape[2]), dtype=np.float64)
    lse = np.zeros((Hq, T), dtype=np.float64)
    for s, (r0, r1) in enumerate(_spans(cu)):
        if r1 == r0:
            continue
        res = fp8_model(qc[None, r0:r1], kc[None, r0:r1], vc[None, r0:r1], q_s[s:s + 1], k_s[s:s + 1],
                        v_s[s:s + 1], rescale_log2=rescale_log2, p_mode=p_mode, return_lse=return_lse,
                        kv_tile=kv_tile)
        if return_lse:
            o[r0:r1] = res[0][0]
            lse[:, r0:r1] = res[1][0]
        else:
            o[r0:r1] = res[0]
    return (o, lse) if return_lse else o


def rel_fro(a, b) -> float:
    """||a - b||_F / ||b||_F in fp64."""
    a = np.asarray(a, dtype=np.float64); b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm((a - b).ravel()) / np.linalg.norm(b.ravel()))
