"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
symbol declared in include/externd.h, and its pure host functions and argument
validation behave as documented."""
import ctypes
import os
import re

import numpy as np
import pytest

import ternary_rank_weight_b200 as ext
from ternary_rank_weight_b200 import _lib
from oracle import externd_oracle as ora

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "externd.h")).read()
    return sorted(set(re.findall(r"\b(externd_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    L = _lib.load()
    declared = _declared_symbols()
    assert declared, "no declarations found"
    for name in declared:
        assert hasattr(L, name), name
    assert set(declared) == set(_lib.EXPORTS)


def test_rank_matches_oracle_rounding():
    for m, n, mu in [(256, 256, 2.0), (2560, 6912, 3.0), (1536, 1536, 2.5), (4096, 4096, 3.5),
                     (3, 5, 0.5), (3, 5, 0.1), (7, 9, 1.2345), (1, 1, 1.0), (0, 5, 1.0), (5, 5, float("nan"))]:
        assert ext.rank(m, n, mu) == ora.rank(m, n, mu), (m, n, mu)


def test_trit_bytes():
    assert ext.trit_bytes(0) == 0
    assert ext.trit_bytes(1) == 16
    assert ext.trit_bytes(64) == 16
    assert ext.trit_bytes(65) == 32
    assert ext.trit_bytes(2560) == 640
    assert ext.trit_bytes(6912) == 1728


def test_trit_codec_round_trip_and_layout():
    rng = np.random.default_rng(0)
    for length in (1, 3, 4, 5, 63, 64, 65, 1000):
        t = rng.integers(-1, 2, size=(3, length)).astype(np.int8)
        p = ext.pack_trits(t)
        assert p.shape == (3, ext.trit_bytes(length))
        assert np.array_equal(ext.unpack_trits(p, length), t)
    # trit j in byte j/4, bits 2*(j%4); 01 = +1, 11 = -1
    p = ext.pack_trits(np.array([[1, 0, -1, 1, -1]], dtype=np.int8))
    assert p[0, 0] == 0b01_11_00_01 and p[0, 1] == 0b11
    assert np.all(p[0, 2:] == 0)


def test_status_strings():
    for s in range(-8, 1):
        assert ext.strerror(s) and ext.strerror(s) != "unknown status"


def test_argument_validation_before_any_device_work():
    L = _lib.load()
    buf = (ctypes.c_uint8 * 64)()
    A = (ctypes.c_float * 4)(1, 2, 3, 4)
    args_ok = dict(A=ctypes.addressof(A), m=2, n=2, mu=1.0, tau=0.7, iters=15)
    def call(**kw):
        a = dict(args_ok, **kw)
        return L.externd_factor(a["A"], a["m"], a["n"], a["mu"], a["tau"], a["iters"], 0,
                                ctypes.addressof(buf), ctypes.addressof(buf), ctypes.addressof(buf), None, None)
    einval = ext.STATUS["EINVAL"]
    assert call(A=None) == einval
    assert call(m=0) == einval
    assert call(n=-3) == einval
    assert call(iters=0) == einval
    assert call(tau=-0.1) == einval
    assert call(tau=float("inf")) == einval
    assert call(mu=float("nan")) == einval
    assert call(mu=0.1) == einval            # k rounds to 0
    assert L.externd_reconstruct(None, None, None, 1, 1, 1, None, None) == einval
    assert L.externd_debug_halfstep(None, 1, 1, 1, None, 0.7, None, None, None, None) == einval
    assert L.externd_factor_batched(0, None, None, None, None, None, 15, None, None, None, None, None, None,
                                    None) == einval


def test_inference_entry_points_reject_bad_arguments_before_device_work():
    L = _lib.load()
    einval = ext.STATUS["EINVAL"]
    host = (ctypes.c_uint8 * 64)()
    p = ctypes.addressof(host)
    assert L.externd_transpose_trits(None, 1, 1, p, None) == einval
    assert L.externd_transpose_trits(p, 0, 1, p, None) == einval
    assert L.externd_transpose_trits(p, 4, 4, p, None) == einval          # host memory is refused
    assert L.externd_matvec(None, p, p, 1, 1, 1, p, 1, p, p, None) == einval
    assert L.externd_matvec(p, p, p, 1, 1, 1, p, 0, p, p, None) == einval   # batch < 1
    assert L.externd_matvec(p, p, p, 2, 2, 2, p, 1, p, p, None) == einval   # host memory is refused
    assert L.externd_pack_mask_sign(p, 1, 1, p, p, 0, p, None) == einval    # no room for signs
    assert L.externd_pack_mask_sign(None, 1, 1, p, p, 1, p, None) == einval


def _c_layout(struct, fields):
    """sizeof and offsetof of a struct of include/externd.h, from the C compiler."""
    import shutil
    import subprocess
    import tempfile
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    body = "".join(f'    printf("%zu\\n", offsetof({struct}, {f}));\n' for f in fields)
    src = ("#include <stddef.h>\n#include <stdio.h>\n#include \"externd.h\"\nint main(void) {\n"
           f'    printf("%zu\\n", sizeof({struct}));\n{body}    return 0;\n}}\n')
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "layout.c")
        exe = os.path.join(d, "layout")
        open(c, "w").write(src)
        subprocess.run([cc, "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        out = [int(x) for x in subprocess.run([exe], check=True, capture_output=True, text=True).stdout.split()]
    return out[0], out[1:]


@pytest.mark.parametrize("cls,struct,rename", [(_lib.Options, "externd_options", {"lambda_": "lambda"}),
                                               (_lib.Stats, "externd_stats", {}),
                                               (_lib.BatchOptions, "externd_batch_options", {"lambda_": "lambda"})])
def test_ctypes_structs_match_the_header(cls, struct, rename):
    names = [n for n, _ in cls._fields_]
    size, offs = _c_layout(struct, [rename.get(n, n) for n in names])
    assert ctypes.sizeof(cls) == size
    for n, off in zip(names, offs):
        assert getattr(cls, n).offset == off, n


def test_factor_options_are_validated_before_device_work():
    L = _lib.load()
    buf = (ctypes.c_uint8 * 64)()
    A = (ctypes.c_float * 4)(1, 2, 3, 4)
    h = (ctypes.c_float * 2)(1, 1)
    einval = ext.STATUS["EINVAL"]
    for kw in ({"sweeps": -1}, {"sweeps": 1001}, {"h": ctypes.addressof(h), "lambda_": -1.0},
               {"h": ctypes.addressof(h), "lambda_": float("nan")}):
        opt = _lib.Options()
        for k, v in kw.items():
            setattr(opt, k, v)
        rc = L.externd_factor_ex(ctypes.addressof(A), 2, 2, 1.0, 0.7, 15, 0, ctypes.addressof(buf),
                                 ctypes.addressof(buf), ctypes.addressof(buf), None, None, ctypes.byref(opt))
        assert rc == einval, kw


def test_batched_options_are_validated_before_device_work():
    L = _lib.load()
    einval = ext.STATUS["EINVAL"]
    buf = (ctypes.c_uint8 * 64)()
    A = (ctypes.c_float * 4)(1, 2, 3, 4)
    h = (ctypes.c_float * 2)(1, 1)
    P2 = ctypes.c_void_p * 2
    a = P2(ctypes.addressof(A), ctypes.addressof(A))
    bp = P2(ctypes.addressof(buf), ctypes.addressof(buf))
    m = (ctypes.c_int64 * 2)(2, 2)
    mu = (ctypes.c_double * 2)(1.0, 1.0)
    tau = (ctypes.c_double * 2)(0.7, 0.7)
    seed = (ctypes.c_uint64 * 2)(0, 1)
    for kw in ({"h": P2(ctypes.addressof(h), None)},                 # weights for one matrix only
               {"h": P2(ctypes.addressof(h), ctypes.addressof(h)), "lambda_": (ctypes.c_double * 2)(0.0, -1.0)},
               {"lambda_": (ctypes.c_double * 2)(0.0, 0.0)},        # lambda without weights
               {"sweeps": -1}, {"sweeps": 1001}):
        opt = _lib.BatchOptions()
        for k, v in kw.items():
            setattr(opt, k, ctypes.cast(v, ctypes.c_void_p) if not isinstance(v, int) else v)
        st = (ctypes.c_int * 2)()
        rc = L.externd_factor_batched_ex(2, a, m, m, mu, tau, 15, seed, bp, bp, bp, None, st, None, ctypes.byref(opt))
        assert rc == einval and list(st) == [einval, einval], kw


def test_binding_rejects_bad_inputs_before_the_library_call():
    import torch
    with pytest.raises(ValueError):
        ext.factor(torch.zeros(3, 4, dtype=torch.float64), 1.0, 0.7)       # not float32
    with pytest.raises(ValueError):
        ext.factor(np.zeros(5, dtype=np.float32), 1.0, 0.7)                # not a matrix
    with pytest.raises(ValueError):
        ext.factor_weighted(np.ones((3, 4), dtype=np.float32), np.ones(3, dtype=np.float32), 1.0, 0.7)
    with pytest.raises(ValueError):
        ext.factor(np.ones((3, 4), dtype=np.float32), 1.0, 0.7, h=np.ones(5, dtype=np.float32))
    with pytest.raises(ext.ExterndError) as e:
        ext.factor(np.ones((3, 4), dtype=np.float32), 0.01, 0.7)          # k rounds to 0
    assert e.value.status == ext.STATUS["EINVAL"]
