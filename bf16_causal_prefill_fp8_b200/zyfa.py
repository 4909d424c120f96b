"""Thin ctypes binding of libzyfa.so (include/zyfa.h) for torch CUDA tensors.

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels.  PyTorch provides device memory and the current stream.  If the
library has not been built, importing the functions raises instead of falling
back to anything else.
"""
import ctypes
import os
import re

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
# ZYFA_CHECKED=1 selects the build with device-side range checks compiled in
LIB_PATH = os.path.join(HERE, "libzyfa_checked.so" if os.environ.get("ZYFA_CHECKED") == "1" else "libzyfa.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "zyfa.h")

BF16, FP8_E4M3, FP32 = 0, 1, 2
OK, ERR_DEVICE_TIMEOUT = 0, -8


class ZyfaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m bf16_causal_prefill_fp8_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        p, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.zyfa_attn_fwd.restype = i
        L.zyfa_attn_fwd.argtypes = [p, p, p, p, i, i, i, i, i, i, i, p, p, p, p]
        L.zyfa_attn_fwd_lse.restype = i
        L.zyfa_attn_fwd_lse.argtypes = [p, p, p, p, p, i, i, i, i, i, i, i, p, p, p, p]
        L.zyfa_attn_fwd_fp8_exact_p.restype = i
        L.zyfa_attn_fwd_fp8_exact_p.argtypes = [p, p, p, p, i, i, i, i, i, i, p, p, p, p]
        L.zyfa_quantize.restype = i
        L.zyfa_quantize.argtypes = [p, i, p, p, i, i, i, i, i, p]
        L.zyfa_quantize_qkv.restype = i
        L.zyfa_quantize_qkv.argtypes = [p, p, p, i, p, p, p, p, p, p, i, i, i, i, i, i, i, p]
        L.zyfa_attn_fwd_varlen.restype = i
        L.zyfa_attn_fwd_varlen.argtypes = [p, p, p, p, p, p, i, i, i, i, i, i, p, p, p, p]
        L.zyfa_quantize_varlen.restype = i
        L.zyfa_quantize_varlen.argtypes = [p, i, p, p, p, i, i, i, i, p]
        L.zyfa_quantize_qkv_varlen.restype = i
        L.zyfa_quantize_qkv_varlen.argtypes = [p, p, p, i, p, p, p, p, p, p, p, i, i, i, i, i, i, p]
        L.zyfa_attn_schedule.restype = i
        L.zyfa_attn_schedule.argtypes = [i, i, p, i, i, i, i, i, i, p, i]
        L.zyfa_attn_kv_tile.restype = i
        L.zyfa_attn_kv_tile.argtypes = [i, i]
        L.zyfa_status_string.restype = ctypes.c_char_p
        L.zyfa_status_string.argtypes = [i]
        L.zyfa_device_status.restype = i
        L.zyfa_device_status.argtypes = [p]
        L.zyfa_set_wait_timeout_ns.restype = None
        L.zyfa_set_wait_timeout_ns.argtypes = [ctypes.c_ulonglong]
        L.zyfa_device_check.restype = i
        L.zyfa_device_check.argtypes = [p]
        L.zyfa_checked_build.restype = i
        L.zyfa_checked_build.argtypes = []
        L.zyfa_leanp_codes.restype = i
        L.zyfa_leanp_codes.argtypes = [p, p, p, p, p, i, p, p, p]
        L.zyfa_selftest_wait_timeout.restype = i
        L.zyfa_selftest_wait_timeout.argtypes = [ctypes.c_ulonglong, p]
        _lib = L
    return _lib


def declared_symbols():
    """Names of the entry points include/zyfa.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?(?:int|void|char\s*\*|const char\s*\*)\s*\**\s*(zyfa_\w+)\s*\(",
                                 text, flags=re.M)))


def status_string(status: int) -> str:
    return lib().zyfa_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != OK:
        raise ZyfaError(status, what)


def _stream(stream=None) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dev(t, name):
    if not (t.is_cuda and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device}, but the current CUDA device is "
                         f"cuda:{torch.cuda.current_device()} (the library launches there)")


# --- argument checks ----------------------------------------------------------
# Shapes, dtypes and devices of every tensor a call passes, checked before the
# library sees a pointer: a wrong extent would let a copy or a store run past
# an allocation.  They take any tensor-like object (the CPU tests pass meta
# tensors); _dev() adds the CUDA and current-device checks at call time.

FP8_DTYPES = (torch.uint8, torch.float8_e4m3fn)


def _want(cond, msg):
    if not cond:
        raise ValueError(msg)


def _same_device(ref, named):
    for t, n in named:
        if t is not None and not isinstance(t, bool):
            _want(t.device == ref.device, f"{n} is on {t.device}, q on {ref.device}")


def _scale_check(t, n, count):
    if t is not None:
        _want(t.dtype == torch.float32, f"{n} must be fp32")
        _want(t.numel() == count, f"{n} holds {t.numel()} values, expected {count} (one per batch entry and head)")


def check_attn_args(q, k, v, o=None, q_scale=None, k_scale=None, v_scale=None, lse=None):
    """attn_fwd's tensors: q [B,S,Hq,Dqk], k [B,S,Hkv,Dqk], v [B,S,Hkv,Dv] of one
    dtype; o bf16 [B,S,Hq,Dv]; lse fp32 [B,Hq,S]; scales fp32 with B*H values;
    all on q's device.  Returns (B, S, Hq, Hkv, Dqk, Dv, dtype code)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _want(t.dim() == 4, f"{n} must be 4-D [B, S, H, D], got {tuple(t.shape)}")
    B, S, Hq, Dqk = q.shape
    Hkv, Dv = k.shape[2], v.shape[3]
    _want(tuple(k.shape) == (B, S, Hkv, Dqk), f"k is {tuple(k.shape)}, expected (B, S, Hkv, Dqk) = {(B, S, Hkv, Dqk)}")
    _want(tuple(v.shape[:3]) == (B, S, Hkv), f"v is {tuple(v.shape)}, expected (B, S, Hkv, Dv) with {(B, S, Hkv)}")
    _want(q.dtype == k.dtype == v.dtype, f"q, k, v dtypes differ: {q.dtype}, {k.dtype}, {v.dtype}")
    if q.dtype == torch.bfloat16:
        dt = BF16
    elif q.dtype in FP8_DTYPES:
        dt = FP8_E4M3
    else:
        raise ValueError(f"unsupported dtype {q.dtype}")
    if o is not None:
        _want(o.dtype == torch.bfloat16 and tuple(o.shape) == (B, S, Hq, Dv),
              f"o must be bf16 [B, S, Hq, Dv] = {(B, S, Hq, Dv)}, got {o.dtype} {tuple(o.shape)}")
    if lse is not None and not isinstance(lse, bool):
        _want(lse.dtype == torch.float32 and tuple(lse.shape) == (B, Hq, S),
              f"lse must be fp32 [B, Hq, S] = {(B, Hq, S)}, got {lse.dtype} {tuple(lse.shape)}")
    for t, n, c in ((q_scale, "q_scale", B * Hq), (k_scale, "k_scale", B * Hkv), (v_scale, "v_scale", B * Hkv)):
        _scale_check(t, n, c)
    _same_device(q, ((k, "k"), (v, "v"), (o, "o"), (lse, "lse"), (q_scale, "q_scale"), (k_scale, "k_scale"),
                     (v_scale, "v_scale")))
    return B, S, Hq, Hkv, Dqk, Dv, dt


def check_quantize_args(x, out=None, scale=None, rows_first=False):
    """quantize's tensors: x bf16 / fp32 [B,S,H,D] (or packed [T,H,D] with
    rows_first), out uint8 / e4m3 of x's shape, scale fp32 (its count is
    checked by the caller, which knows B or the sequence count)."""
    _want(x.dim() == (3 if rows_first else 4), f"x has {x.dim()} dimensions")
    _want(x.dtype in (torch.bfloat16, torch.float32), f"unsupported input dtype {x.dtype}")
    if out is not None:
        _want(tuple(out.shape) == tuple(x.shape) and out.dtype in FP8_DTYPES,
              f"out must be uint8 / float8_e4m3fn of x's shape {tuple(x.shape)}, got {out.dtype} {tuple(out.shape)}")
    if scale is not None:
        _want(scale.dtype == torch.float32, "scale must be fp32")
    _same_device(x, ((out, "out"), (scale, "scale")))


def check_varlen_args(q, k, v, T, nseq, o=None, q_scale=None, k_scale=None, v_scale=None, lse=None):
    """attn_fwd_varlen's tensors: packed q [T,Hq,Dqk], k [T,Hkv,Dqk], v [T,Hkv,Dv]
    of one dtype; o bf16 [T,Hq,Dv]; lse fp32 [Hq,T]; scales fp32 with nseq*H
    values; all on q's device."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _want(t.dim() == 3, f"{n} must be 3-D [T, H, D], got {tuple(t.shape)}")
        _want(t.shape[0] == T, f"{n} holds {t.shape[0]} rows, cu_seqlens[-1] = {T}")
    _, Hq, Dqk = q.shape
    Hkv, Dv = k.shape[1], v.shape[2]
    _want(k.shape[2] == Dqk and v.shape[1] == Hkv, f"k {tuple(k.shape)} / v {tuple(v.shape)} do not match q {tuple(q.shape)}")
    _want(q.dtype == k.dtype == v.dtype, f"q, k, v dtypes differ: {q.dtype}, {k.dtype}, {v.dtype}")
    if o is not None:
        _want(o.dtype == torch.bfloat16 and tuple(o.shape) == (T, Hq, Dv),
              f"o must be bf16 [T, Hq, Dv] = {(T, Hq, Dv)}, got {o.dtype} {tuple(o.shape)}")
    if lse is not None and not isinstance(lse, bool):
        _want(lse.dtype == torch.float32 and tuple(lse.shape) == (Hq, T), f"lse must be fp32 [Hq, T] = {(Hq, T)}")
    for t, n, c in ((q_scale, "q_scale", nseq * Hq), (k_scale, "k_scale", nseq * Hkv), (v_scale, "v_scale", nseq * Hkv)):
        _scale_check(t, n, c)
    _same_device(q, ((k, "k"), (v, "v"), (o, "o"), (lse, "lse"), (q_scale, "q_scale"), (k_scale, "k_scale"),
                     (v_scale, "v_scale")))


def attn_fwd(q, k, v, o=None, q_scale=None, k_scale=None, v_scale=None, stream=None, exact_p=False, lse=False):
    """Causal attention forward.  q [B,S,Hq,Dqk], k [B,S,Hkv,Dqk], v [B,S,Hkv,Dv];
    bf16 tensors (BF16 path) or uint8 / float8_e4m3fn codes with fp32 scales
    [B,H] (FP8 path).  exact_p (FP8 only): the exact-P ablation
    (zyfa_attn_fwd_fp8_exact_p) instead of Lean P.  Returns o [B,S,Hq,Dv] bf16;
    with lse=True (or an fp32 [B,Hq,S] tensor) returns (o, lse) through
    zyfa_attn_fwd_lse."""
    B, S, Hq, Hkv, Dqk, Dv, dt = check_attn_args(q, k, v, o, q_scale, k_scale, v_scale, lse)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, n)
    if o is None:
        o = torch.empty((B, S, Hq, Dv), dtype=torch.bfloat16, device=q.device)
    _dev(o, "o")
    for t, n in ((q_scale, "q_scale"), (k_scale, "k_scale"), (v_scale, "v_scale")):
        if t is not None:
            _dev(t, n)
    if lse is not False and lse is not None:
        if exact_p:
            raise ValueError("lse is not produced by the exact-P ablation")
        out = torch.empty((B, Hq, S), dtype=torch.float32, device=q.device) if lse is True else lse
        _dev(out, "lse")
        st = lib().zyfa_attn_fwd_lse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(out), B, Hq, Hkv, S, Dqk, Dv, dt,
                                     _ptr(q_scale), _ptr(k_scale), _ptr(v_scale), _stream(stream))
        _check(st, "zyfa_attn_fwd_lse")
        return o, out
    if exact_p:
        if dt != FP8_E4M3:
            raise ValueError("exact_p applies to the FP8 path only")
        st = lib().zyfa_attn_fwd_fp8_exact_p(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Hq, Hkv, S, Dqk, Dv,
                                             _ptr(q_scale), _ptr(k_scale), _ptr(v_scale), _stream(stream))
        _check(st, "zyfa_attn_fwd_fp8_exact_p")
        return o
    st = lib().zyfa_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Hq, Hkv, S, Dqk, Dv, dt,
                             _ptr(q_scale), _ptr(k_scale), _ptr(v_scale), _stream(stream))
    _check(st, "zyfa_attn_fwd")
    return o


def quantize(x, hadamard=False, out=None, scale=None, stream=None):
    """x [B,S,H,D] bf16 or fp32 -> (codes uint8 [B,S,H,D], scale fp32 [B,H])."""
    check_quantize_args(x, out, scale)
    _dev(x, "x")
    dt = BF16 if x.dtype == torch.bfloat16 else FP32
    B, S, H, D = x.shape
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if scale is None:
        scale = torch.empty((B, H), dtype=torch.float32, device=x.device)
    _scale_check(scale, "scale", B * H)
    _dev(out, "out"); _dev(scale, "scale")
    st = lib().zyfa_quantize(_ptr(x), dt, _ptr(out), _ptr(scale), B, S, H, D, int(bool(hadamard)),
                             _stream(stream))
    _check(st, "zyfa_quantize")
    return out, scale


def quantize_qkv(q, k, v, hadamard_qk=False, out=None, stream=None):
    """Q, K, V [B,S,H,D] (same dtype: bf16 or fp32) -> ((q8, q_scale), (k8, k_scale), (v8, v_scale)),
    identical to three quantize() calls (Hadamard on Q and K only), in four launches.  `out`: optional
    ((q8, qs), (k8, ks), (v8, vs)) to write into."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        check_quantize_args(t)
    _want(q.dtype == k.dtype == v.dtype, "q, k and v must share a dtype")
    _want(k.shape[:2] == q.shape[:2] and v.shape[:3] == k.shape[:3] and k.shape[3] == q.shape[3],
          f"q {tuple(q.shape)}, k {tuple(k.shape)}, v {tuple(v.shape)} do not form one problem")
    _same_device(q, ((k, "k"), (v, "v")))
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, n)
    dt = BF16 if q.dtype == torch.bfloat16 else FP32
    B, S, Hq, Dqk = q.shape
    Hkv, Dv = k.shape[2], v.shape[3]
    if out is None:
        out = tuple((torch.empty(t.shape, dtype=torch.uint8, device=t.device),
                     torch.empty((B, t.shape[2]), dtype=torch.float32, device=t.device)) for t in (q, k, v))
    for (c, sc), x, n in zip(out, (q, k, v), "qkv"):
        check_quantize_args(x, c, sc)
        _scale_check(sc, n + "_scale", B * x.shape[2])
        _dev(c, n + "_fp8"); _dev(sc, n + "_scale")
    (q8, qs), (k8, ks), (v8, vs) = out
    st = lib().zyfa_quantize_qkv(_ptr(q), _ptr(k), _ptr(v), dt, _ptr(q8), _ptr(k8), _ptr(v8), _ptr(qs), _ptr(ks),
                                 _ptr(vs), B, S, Hq, Hkv, Dqk, Dv, int(bool(hadamard_qk)), _stream(stream))
    _check(st, "zyfa_quantize_qkv")
    return out


def _cu_host(cu_seqlens, rows=None):
    """cu_seqlens (list, numpy array or CPU tensor of nseq + 1 ints) -> (ctypes int array, nseq).
    rows: the packed tensors' row count, which must equal cu_seqlens[-1]."""
    if isinstance(cu_seqlens, torch.Tensor):
        if cu_seqlens.is_cuda:
            raise ValueError("cu_seqlens must be host memory (a CPU tensor or a list)")
        cu_seqlens = cu_seqlens.tolist()
    vals = [int(x) for x in cu_seqlens]
    if len(vals) < 2:
        raise ValueError("cu_seqlens needs nseq + 1 >= 2 entries")
    if rows is not None and vals[-1] != rows:
        raise ValueError(f"cu_seqlens[-1] = {vals[-1]} but the packed tensors hold {rows} rows")
    return (ctypes.c_int * len(vals))(*vals), len(vals) - 1


def attn_fwd_varlen(q, k, v, cu_seqlens, o=None, q_scale=None, k_scale=None, v_scale=None, lse=False,
                    stream=None):
    """Causal attention over a packed batch (zyfa_attn_fwd_varlen).  q [T,Hq,Dqk], k [T,Hkv,Dqk],
    v [T,Hkv,Dv] with sequence s at rows cu_seqlens[s] .. cu_seqlens[s+1]-1; bf16, or e4m3 codes
    with fp32 scales [nseq,H].  Returns o [T,Hq,Dv] bf16, or (o, lse [Hq,T] fp32) with lse=True
    (or an fp32 [Hq,T] tensor)."""
    if q.dtype == torch.bfloat16:
        dt = BF16
    elif q.dtype in FP8_DTYPES:
        dt = FP8_E4M3
    else:
        raise ValueError(f"unsupported dtype {q.dtype}")
    T = q.shape[0]
    cu, nseq = _cu_host(cu_seqlens, T)
    check_varlen_args(q, k, v, T, nseq, o, q_scale, k_scale, v_scale, lse)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, n)
    _, Hq, Dqk = q.shape
    Hkv, Dv = k.shape[1], v.shape[2]
    if o is None:
        o = torch.empty((T, Hq, Dv), dtype=torch.bfloat16, device=q.device)
    _dev(o, "o")
    for t, n in ((q_scale, "q_scale"), (k_scale, "k_scale"), (v_scale, "v_scale")):
        if t is not None:
            _dev(t, n)
    out = None
    if lse is not False and lse is not None:
        out = torch.empty((Hq, T), dtype=torch.float32, device=q.device) if lse is True else lse
        _dev(out, "lse")
    st = lib().zyfa_attn_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(out), cu, nseq, Hq, Hkv, Dqk, Dv,
                                    dt, _ptr(q_scale), _ptr(k_scale), _ptr(v_scale), _stream(stream))
    _check(st, "zyfa_attn_fwd_varlen")
    return o if out is None else (o, out)


def _in_dtype(x):
    if x.dtype == torch.bfloat16:
        return BF16
    if x.dtype == torch.float32:
        return FP32
    raise ValueError(f"unsupported input dtype {x.dtype}")


def quantize_varlen(x, cu_seqlens, hadamard=False, out=None, scale=None, stream=None):
    """x [T,H,D] bf16 or fp32, packed -> (codes uint8 [T,H,D], scale fp32 [nseq,H])."""
    check_quantize_args(x, out, scale, rows_first=True)
    _dev(x, "x")
    dt = _in_dtype(x)
    T, H, D = x.shape
    cu, nseq = _cu_host(cu_seqlens, T)
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if scale is None:
        scale = torch.empty((nseq, H), dtype=torch.float32, device=x.device)
    _scale_check(scale, "scale", nseq * H)
    _dev(out, "out"); _dev(scale, "scale")
    st = lib().zyfa_quantize_varlen(_ptr(x), dt, _ptr(out), _ptr(scale), cu, nseq, H, D, int(bool(hadamard)),
                                    _stream(stream))
    _check(st, "zyfa_quantize_varlen")
    return out, scale


def quantize_qkv_varlen(q, k, v, cu_seqlens, hadamard_qk=False, out=None, stream=None):
    """Packed Q, K, V [T,H,D] (same dtype) -> ((q8, q_scale), (k8, k_scale), (v8, v_scale)), scales
    [nseq,H]; identical to three quantize_varlen() calls, in four launches."""
    for t in (q, k, v):
        check_quantize_args(t, rows_first=True)
    _want(q.dtype == k.dtype == v.dtype, "q, k and v must share a dtype")
    dt = _in_dtype(q)
    T, Hq, Dqk = q.shape
    Hkv, Dv = k.shape[1], v.shape[2]
    for t, n in ((k, "k"), (v, "v")):
        if t.shape[0] != T:
            raise ValueError(f"{n} holds {t.shape[0]} rows, q holds {T}")
    _same_device(q, ((k, "k"), (v, "v")))
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, n)
    cu, nseq = _cu_host(cu_seqlens, T)
    if out is None:
        out = tuple((torch.empty(t.shape, dtype=torch.uint8, device=t.device),
                     torch.empty((nseq, t.shape[1]), dtype=torch.float32, device=t.device)) for t in (q, k, v))
    for (c, sc), x, n in zip(out, (q, k, v), "qkv"):
        check_quantize_args(x, c, sc, rows_first=True)
        _scale_check(sc, n + "_scale", nseq * x.shape[1])
        _dev(c, n + "_fp8"); _dev(sc, n + "_scale")
    (q8, qs), (k8, ks), (v8, vs) = out
    st = lib().zyfa_quantize_qkv_varlen(_ptr(q), _ptr(k), _ptr(v), dt, _ptr(q8), _ptr(k8), _ptr(v8), _ptr(qs),
                                        _ptr(ks), _ptr(vs), cu, nseq, Hq, Hkv, Dqk, Dv, int(bool(hadamard_qk)),
                                        _stream(stream))
    _check(st, "zyfa_quantize_qkv_varlen")
    return out


def attn_schedule(Hq, Hkv, Dqk, dtype, grid, cta, B=None, S=None, cu_seqlens=None):
    """Host-only: the (b, hq, qt) units CTA `cta` of a `grid`-CTA launch runs, in order (a list of
    tuples).  Fixed length: B and S; packed batch: cu_seqlens."""
    if cu_seqlens is not None:
        cu, nseq = _cu_host(cu_seqlens)
        B, S = nseq, 0
    else:
        cu = None
    L = lib()
    n = L.zyfa_attn_schedule(B, S, cu, Hq, Hkv, Dqk, dtype, grid, cta, None, 0)
    if n < 0:
        raise ZyfaError(n, "zyfa_attn_schedule")
    buf = (ctypes.c_int * max(1, 3 * n))()
    m = L.zyfa_attn_schedule(B, S, cu, Hq, Hkv, Dqk, dtype, grid, cta, buf, n)
    if m != n:
        raise ZyfaError(m if m < 0 else -2, "zyfa_attn_schedule")
    return [(buf[3 * i], buf[3 * i + 1], buf[3 * i + 2]) for i in range(n)]


def kv_tile(dtype, Dqk) -> int:
    """Host-only: keys per KV tile of the attention kernel run for (dtype, Dqk); the deferred
    reference max is decided once per such tile."""
    n = lib().zyfa_attn_kv_tile(int(dtype), int(Dqk))
    if n < 0:
        raise ZyfaError(n, "zyfa_attn_kv_tile")
    return n


def leanp_codes(s, m, bmax, A, masked=None, stream=None):
    """Element-wise Lean-P codes from the kernel's device functions."""
    n = s.numel()
    for t, nm in ((s, "s"), (m, "m"), (bmax, "bmax"), (A, "A")):
        _dev(t, nm)
    code = torch.empty(n, dtype=torch.uint8, device=s.device)
    j = torch.empty(n, dtype=torch.int32, device=s.device)
    st = lib().zyfa_leanp_codes(_ptr(s), _ptr(m), _ptr(bmax), _ptr(A), _ptr(masked), n, _ptr(code),
                                _ptr(j), _stream(stream))
    _check(st, "zyfa_leanp_codes")
    return code, j


def device_status(stream=None) -> int:
    return lib().zyfa_device_status(_stream(stream))


def device_check(stream=None) -> int:
    """Checked build: site of the first failed range check since the last call (0 = none)."""
    return lib().zyfa_device_check(_stream(stream))


def checked_build() -> bool:
    return bool(lib().zyfa_checked_build())


def set_wait_timeout_ns(ns: int):
    lib().zyfa_set_wait_timeout_ns(int(ns))


def selftest_wait_timeout(ns: int, stream=None):
    _check(lib().zyfa_selftest_wait_timeout(int(ns), _stream(stream)), "zyfa_selftest_wait_timeout")
