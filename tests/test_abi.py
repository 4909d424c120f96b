"""The C-ABI library loads, exports every symbol include/zyfa.h declares, and
rejects bad arguments on the host before touching the GPU (runs without a GPU)."""
import ctypes

import pytest

from bf16_causal_prefill_fp8_b200 import build, zyfa


@pytest.fixture(scope="module")
def L():
    build.build()
    return zyfa.lib()


def test_every_declared_symbol_is_exported(L):
    names = zyfa.declared_symbols()
    assert set(names) >= {"zyfa_attn_fwd", "zyfa_attn_fwd_lse", "zyfa_attn_fwd_fp8_exact_p", "zyfa_quantize",
                          "zyfa_quantize_qkv", "zyfa_attn_fwd_varlen", "zyfa_quantize_varlen",
                          "zyfa_quantize_qkv_varlen", "zyfa_attn_schedule", "zyfa_attn_kv_tile",
                          "zyfa_status_string",
                          "zyfa_device_status",
                          "zyfa_leanp_codes", "zyfa_selftest_wait_timeout", "zyfa_set_wait_timeout_ns"}
    for n in names:
        assert hasattr(L, n), n


def test_kv_tile_per_dtype_and_head_dim(L):
    # FP8 with Dqk 128 runs 256-key KV tiles; the MLA shape and BF16 128-key ones
    assert zyfa.kv_tile(zyfa.FP8_E4M3, 128) == 256
    assert zyfa.kv_tile(zyfa.FP8_E4M3, 192) == 128
    assert zyfa.kv_tile(zyfa.BF16, 128) == 128
    assert zyfa.kv_tile(zyfa.BF16, 192) == 128
    assert L.zyfa_attn_kv_tile(7, 128) < 0
    assert L.zyfa_attn_kv_tile(zyfa.FP8_E4M3, 64) < 0
    with pytest.raises(zyfa.ZyfaError):
        zyfa.kv_tile(zyfa.FP8_E4M3, 256)


def test_status_strings(L):
    for st in [0, -1, -2, -3, -4, -5, -6, -7, -8, 12345]:
        s = zyfa.status_string(st)
        assert isinstance(s, str) and s
    assert zyfa.status_string(0) == "ok"
    assert zyfa.status_string(12345) == "unknown status"


FAKE = 1 << 20  # a 16-byte aligned non-null address; never dereferenced (validation fails first)


def _attn(L, q=FAKE, k=FAKE, v=FAKE, o=FAKE, B=1, Hq=2, Hkv=2, S=128, Dqk=128, Dv=128, dt=0,
          qs=None, ks=None, vs=None):
    return L.zyfa_attn_fwd(q, k, v, o, B, Hq, Hkv, S, Dqk, Dv, dt, qs, ks, vs, None)


def test_attn_argument_errors(L):
    assert _attn(L, q=None) == -1
    assert _attn(L, o=None) == -1
    assert _attn(L, B=0) == -2
    assert _attn(L, S=0) == -2
    assert _attn(L, Hq=0) == -2
    assert _attn(L, Hq=3, Hkv=2) == -4
    assert _attn(L, Dqk=64) == -3
    assert _attn(L, Dqk=128, Dv=64) == -3
    assert _attn(L, Dqk=192, Dv=192) == -3
    assert _attn(L, dt=2) == -6
    assert _attn(L, dt=-1) == -6
    assert _attn(L, q=FAKE + 8) == -5
    assert _attn(L, o=FAKE + 2) == -5
    assert _attn(L, dt=1, qs=FAKE + 1) == -5
    assert _attn(L, B=1 << 20, Hq=1 << 12, Hkv=1, S=1 << 16) == -2


def test_lse_argument_errors(L):
    def e(lse=FAKE, q=FAKE, B=1, S=128, dt=0):
        return L.zyfa_attn_fwd_lse(q, FAKE, FAKE, FAKE, lse, B, 2, 2, S, 128, 128, dt, None, None, None, None)
    assert e(lse=None) == -1
    assert e(q=None) == -1
    assert e(lse=FAKE + 2) == -5
    assert e(S=0) == -2
    assert e(dt=3) == -6


def test_exact_p_argument_errors(L):
    def e(q=FAKE, o=FAKE, B=1, Hq=2, Hkv=2, S=128, Dqk=128, Dv=128, qs=None):
        return L.zyfa_attn_fwd_fp8_exact_p(q, FAKE, FAKE, o, B, Hq, Hkv, S, Dqk, Dv, qs, None, None, None)
    assert e(q=None) == -1
    assert e(S=0) == -2
    assert e(Hq=3) == -4
    assert e(Dqk=64) == -3
    assert e(o=FAKE + 4) == -5
    assert e(qs=FAKE + 2) == -5


def test_quantize_argument_errors(L):
    def q(x=FAKE, dt=0, out=FAKE, sc=FAKE, B=1, S=16, H=2, D=128, had=0):
        return L.zyfa_quantize(x, dt, out, sc, B, S, H, D, had, None)
    assert q(x=None) == -1
    assert q(sc=None) == -1
    assert q(B=0) == -2
    assert q(H=5000) == -2
    assert q(dt=1) == -6
    assert q(had=2) == -6
    assert q(D=12) == -3
    assert q(D=64, had=1) == -3
    assert q(D=256, had=1) == -3
    assert q(x=FAKE + 4) == -5
    assert q(sc=FAKE + 2) == -5


def test_quantize_qkv_argument_errors(L):
    def q(q=FAKE, k=FAKE, v=FAKE, dt=0, q8=FAKE, k8=FAKE, v8=FAKE, qs=FAKE, ks=FAKE, vs=FAKE, B=1, S=16, Hq=4,
          Hkv=2, Dqk=128, Dv=128, had=0):
        return L.zyfa_quantize_qkv(q, k, v, dt, q8, k8, v8, qs, ks, vs, B, S, Hq, Hkv, Dqk, Dv, had, None)
    assert q(v=None) == -1
    assert q(ks=None) == -1
    assert q(S=0) == -2
    assert q(Hkv=0) == -2
    assert q(dt=1) == -6
    assert q(had=3) == -6
    assert q(Dv=4) == -3
    assert q(Dqk=64, had=1) == -3
    assert q(k8=FAKE + 8) == -5
    assert q(vs=FAKE + 1) == -5


def test_leanp_and_selftest_argument_errors(L):
    assert L.zyfa_leanp_codes(None, None, None, None, None, -1, None, None, None) == -2
    assert L.zyfa_leanp_codes(None, None, None, None, None, 0, None, None, None) == 0
    assert L.zyfa_leanp_codes(None, FAKE, FAKE, FAKE, None, 4, FAKE, None, None) == -1
    assert L.zyfa_selftest_wait_timeout(ctypes.c_ulonglong(2_000_000_000), None) == -2


def _cu(vals):
    return (ctypes.c_int * len(vals))(*vals)


def test_varlen_argument_errors(L):
    def e(cu=(0, 100, 300), nseq=None, q=FAKE, o=FAKE, lse=None, Hq=2, Hkv=2, Dqk=128, Dv=128, dt=0, qs=None):
        c = None if cu is None else _cu(cu)
        n = (len(cu) - 1) if nseq is None else nseq
        return L.zyfa_attn_fwd_varlen(q, FAKE, FAKE, o, lse, c, n, Hq, Hkv, Dqk, Dv, dt, qs, None, None, None)
    assert e(cu=None, nseq=2) == -1
    assert e(q=None) == -1
    assert e(nseq=0) == -2
    assert e(cu=[0] * 386) == -2                      # more than 384 sequences
    assert e(cu=(1, 100, 300)) == -2                  # cu[0] != 0
    assert e(cu=(0, 300, 100)) == -2                  # decreasing
    assert e(Hq=3) == -4
    assert e(Dqk=64) == -3
    assert e(dt=2) == -6
    assert e(q=FAKE + 8) == -5
    assert e(lse=FAKE + 2) == -5
    assert e(dt=1, qs=FAKE + 1) == -5
    assert e(cu=(0, 0, 0)) == 0                       # every sequence empty: nothing to launch
    assert e(cu=[0] * 385) == 0                       # 384 empty sequences
    assert e(cu=(0, 0), q=None, o=None) == 0          # nothing to read or write
    assert e(cu=(0, 0), Hq=3) == -4


def test_quantize_varlen_argument_errors(L):
    def e(cu=(0, 10, 30), nseq=None, x=FAKE, H=2, D=128, had=0, dt=0):
        c = None if cu is None else _cu(cu)
        n = (len(cu) - 1) if nseq is None else nseq
        return L.zyfa_quantize_varlen(x, dt, FAKE, FAKE, c, n, H, D, had, None)
    assert e(x=None) == -1
    assert e(cu=None, nseq=2) == -1
    assert e(nseq=0) == -2
    assert e(cu=(0, 5, 4)) == -2
    assert e(cu=[0] * 386) == -2
    assert e(H=0) == -2
    assert e(D=100) == -3
    assert e(D=64, had=1) == -3
    assert e(dt=1) == -6
    assert e(had=2) == -6
    assert e(x=FAKE + 4) == -5

    def e3(cu=(0, 10, 30), Hq=4, Hkv=2, Dqk=192, Dv=128, had=1):
        c = _cu(cu)
        return L.zyfa_quantize_qkv_varlen(FAKE, FAKE, FAKE, 0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, c, len(cu) - 1,
                                          Hq, Hkv, Dqk, Dv, had, None)
    assert e3(cu=(0, 10, 3)) == -2
    assert e3(Hkv=0) == -2
    assert e3(Dqk=64) == -3
    assert e3(Dv=12) == -3
    assert e3(had=3) == -6


def test_binding_fails_loudly_without_the_library(monkeypatch):
    """No fallback: with the shared library absent, the first call raises."""
    monkeypatch.setattr(zyfa, "LIB_PATH", zyfa.LIB_PATH + ".absent")
    monkeypatch.setattr(zyfa, "_lib", None)
    with pytest.raises(ImportError):
        zyfa.lib()
    with pytest.raises(ImportError):
        zyfa.status_string(0)


def test_product_package_never_touches_the_oracle():
    """The oracle is test infrastructure: nothing in the package imports it."""
    import os
    import re
    pkg = os.path.dirname(zyfa.__file__)
    for root, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(root, f), encoding="utf-8").read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, flags=re.M), f
                assert "oracle.c" not in text and "liboracle" not in text, f


def test_oracle_uses_nothing_from_the_package():
    """The other direction: the oracle includes only the C library and imports
    neither the package nor its headers."""
    import os
    import re
    here = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    odir = os.path.join(here, "oracle")
    for f in os.listdir(odir):
        path = os.path.join(odir, f)
        if f.endswith(".c"):
            incs = re.findall(r'^\s*#\s*include\s*[<"]([^>"]+)[>"]', open(path).read(), flags=re.M)
            assert set(incs) <= {"math.h", "stdint.h", "stdlib.h", "string.h", "omp.h"}, (f, incs)
        elif f.endswith(".py"):
            imports = re.findall(r"^\s*(?:import|from)\s+([\w.]+)", open(path).read(), flags=re.M)
            assert not any(m.startswith("bf16_causal_prefill_fp8_b200") for m in imports), (f, imports)
            assert "libzyfa" not in open(path).read(), f


def test_checked_build_exports_the_same_symbols():
    """libzyfa_checked.so (device-side range checks compiled in) has the same
    C ABI; each library reports which build it is."""
    Lc = ctypes.CDLL(build.LIB_CHECKED)
    for n in zyfa.declared_symbols():
        assert hasattr(Lc, n), n
    Lc.zyfa_checked_build.restype = ctypes.c_int
    assert Lc.zyfa_checked_build() == 1
    assert zyfa.lib().zyfa_checked_build() == 0


# --- the binding's argument checks (meta tensors: shapes, dtypes and devices only)

def _meta(shape, dtype=None):
    import torch
    return torch.empty(shape, dtype=dtype or torch.bfloat16, device="meta")


def test_binding_rejects_mismatched_attention_tensors():
    import torch
    q, k, v = _meta((2, 256, 4, 128)), _meta((2, 256, 2, 128)), _meta((2, 256, 2, 128))
    assert zyfa.check_attn_args(q, k, v) == (2, 256, 4, 2, 128, 128, zyfa.BF16)
    u8 = lambda *s: _meta(s, torch.uint8)
    f32 = lambda *s: _meta(s, torch.float32)
    assert zyfa.check_attn_args(u8(2, 256, 4, 192), u8(2, 256, 2, 192), u8(2, 256, 2, 128),
                                q_scale=f32(2, 4), k_scale=f32(4), v_scale=f32(2, 2))[6] == zyfa.FP8_E4M3
    bad = [dict(k=_meta((2, 255, 2, 128))),                 # S differs
           dict(k=_meta((1, 256, 2, 128))),                 # B differs
           dict(k=_meta((2, 256, 2, 64))),                  # Dqk differs
           dict(v=_meta((2, 256, 3, 128))),                 # Hkv differs
           dict(v=_meta((2, 256, 2, 128), torch.float32)),  # dtype differs
           dict(q=_meta((2, 256, 4, 128), torch.float16), k=_meta((2, 256, 2, 128), torch.float16),
                v=_meta((2, 256, 2, 128), torch.float16)),  # unsupported dtype
           dict(k=_meta((2, 256, 128))),                    # not 4-D
           dict(o=_meta((2, 256, 4, 64))),                  # o shape
           dict(o=_meta((2, 256, 4, 128), torch.float32)),  # o dtype
           dict(lse=f32(2, 4, 255)), dict(lse=_meta((2, 4, 256))),
           dict(q_scale=f32(3)), dict(k_scale=f32(2, 4)), dict(v_scale=_meta((4,)))]
    for case in bad:
        args = dict(q=q, k=k, v=v)
        args.update(case)
        with pytest.raises(ValueError):
            zyfa.check_attn_args(**args)
    # every tensor on q's device
    with pytest.raises(ValueError):
        zyfa.check_attn_args(q, k, torch.empty((2, 256, 2, 128), dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        zyfa.check_attn_args(q, k, v, o=torch.empty((2, 256, 4, 128), dtype=torch.bfloat16))


def test_binding_rejects_mismatched_prepass_and_packed_tensors():
    import torch
    x = _meta((1, 128, 8, 128))
    zyfa.check_quantize_args(x, _meta((1, 128, 8, 128), torch.uint8), _meta((1, 8), torch.float32))
    for out, scale in ((_meta((1, 128, 8, 64), torch.uint8), None), (_meta((1, 128, 8, 128)), None),
                       (None, _meta((8,)))):
        with pytest.raises(ValueError):
            zyfa.check_quantize_args(x, out, scale)
    with pytest.raises(ValueError):
        zyfa.check_quantize_args(_meta((1, 128, 8, 128), torch.float16))
    with pytest.raises(ValueError):
        zyfa._scale_check(_meta((7,), torch.float32), "scale", 8)
    q, k, v = _meta((300, 4, 128)), _meta((300, 2, 128)), _meta((300, 2, 128))
    zyfa.check_varlen_args(q, k, v, 300, 3, o=_meta((300, 4, 128)), lse=_meta((4, 300), torch.float32))
    for case in (dict(T=299), dict(k=_meta((300, 2, 64))), dict(v=_meta((300, 3, 128))),
                 dict(o=_meta((300, 4, 64))), dict(lse=_meta((300, 4), torch.float32)),
                 dict(q_scale=_meta((4,), torch.float32))):
        args = dict(q=q, k=k, v=v, T=300, nseq=3)
        args.update(case)
        with pytest.raises(ValueError):
            zyfa.check_varlen_args(**args)


def test_binding_refuses_host_tensors_before_any_launch():
    import torch
    q = torch.zeros((1, 128, 2, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        zyfa.attn_fwd(q, q, q)
    with pytest.raises(ValueError):
        zyfa.quantize(q)
