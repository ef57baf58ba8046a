"""Host-side checks of the C ABI: the library loads, exports every symbol the
header declares, carries the oracle's NF4 book bit for bit, and rejects bad
arguments before touching the device.  No kernel is launched here."""
import ctypes
import os
import re

import numpy as np
import pytest

from bit_nf4_quantized_07_b200 import api
from oracle import codec

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", fn)).read()
        names |= set(re.findall(r"QLN_API\s+[\w\s\*]+?\b(\w+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def L():
    from bit_nf4_quantized_07_b200 import build
    build.build()
    return api.lib()


def test_every_declared_symbol_is_exported(L):
    declared = _declared_symbols()
    assert declared == set(api.EXPORTS), declared
    for name in declared:
        assert hasattr(L, name), name


def test_only_the_abi_is_exported(L):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", api.LIB_PATH], capture_output=True, text=True).stdout
    text = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert text == set(api.EXPORTS)


def test_library_codebook_equals_oracle_construction(L):
    lib_cb = api.codebook().numpy()
    _, ora = codec.codebook()
    assert np.array_equal(lib_cb.view(np.uint32), ora.view(np.uint32))


def test_version_and_status_strings(L):
    assert api.version() >> 16 == 1
    for code, name in api.STATUS_NAMES.items():
        assert api.status_str(code) == name


def test_workspace_sizes(L):
    # double quantization: a 256-byte header (status, barrier counters, the
    # exact sum of mu) whatever nb is
    assert api.workspace_bytes(api.OP_DOUBLE_QUANT, 4096) == 256
    assert api.workspace_bytes(api.OP_DOUBLE_QUANT, 1 << 25) == 256
    assert api.workspace_bytes(api.OP_DOUBLE_QUANT, 0) == 0
    f = api.workspace_bytes(api.OP_LINEAR_FWD, 11008, 4096, 2048, 16)
    assert f >= 256 + 2 * 2048 * 16 * 2
    b = api.workspace_bytes(api.OP_LINEAR_BWD, 11008, 4096, 2048, 16)
    assert b >= 256 + 11008 * 16 * 2 + 3 * 2048 * 16 * 2
    assert api.workspace_bytes(99, 1, 1, 1, 1) == 0
    for v in (f, b, api.workspace_bytes(api.OP_DOUBLE_QUANT, 1)):
        assert v % 256 == 0


# Argument errors are reported before any CUDA call, so they can be checked
# with fake, never-dereferenced addresses on a machine without a GPU.
P = ctypes.c_void_p
A16 = P(0x10000)          # 16-byte aligned fake device address
A4 = P(0x10004)           # 4-byte aligned only


def _w(codes=A16, absmax=A16, qabs=None, scale=None, mean=None, rows=64, cols=64):
    return api.CNF4Weight(codes.value if codes else None, absmax.value if absmax else None,
                          qabs.value if qabs else None, scale.value if scale else None,
                          mean.value if mean else None, rows, cols)


def test_quantize_argument_errors(L):
    assert L.nf4_quantize(None, 64, A16, A16, None) == 1
    assert L.nf4_quantize(A16, 0, A16, A16, None) == 2
    assert L.nf4_quantize(A16, 96, A16, A16, None) == 2
    assert L.nf4_quantize(A4, 64, A16, A16, None) == 3
    assert L.nf4_quantize(A16, 64, A4, A16, None) == 3


def test_double_quant_argument_errors(L):
    ws = P(0x20000)
    need = api.workspace_bytes(api.OP_DOUBLE_QUANT, 100)
    assert L.nf4_double_quant(None, 100, A16, A16, A16, ws, need, None) == 1
    assert L.nf4_double_quant(A16, 0, A16, A16, A16, ws, need, None) == 2
    assert L.nf4_double_quant(A16, (1 << 25) + 1, A16, A16, A16, ws, 1 << 40, None) == 2
    assert L.nf4_double_quant(A16, 100, A16, A16, A16, P(0x20010), need, None) == 3
    assert L.nf4_double_quant(A16, 100, A16, A16, A16, ws, need - 1, None) == 4


def test_quantize_dq_argument_errors(L):
    ws = P(0x20000)
    q = lambda **k: L.nf4_quantize_dq(k.get("W", A16), k.get("dtype", 0), k.get("numel", 4096), k.get("fmt", 0),
                                      A16, k.get("absmax", A16), A16, A16, A16, k.get("ws", ws),
                                      k.get("wsb", 256), None)
    assert q(W=None) == 1
    assert q(ws=None) == 1
    assert q(numel=0) == 2
    assert q(numel=(1 << 31) + 1) == 2
    assert q(dtype=7) == 2
    assert q(fmt=2) == 2
    assert q(W=A4) == 3
    assert q(absmax=A4) == 3            # 16-byte: the group pass reads 8 constants at a time
    assert q(ws=P(0x20010)) == 3
    assert q(wsb=255) == 4


def test_quantize_dq_batch_argument_errors(L):
    ws = P(0x20000)
    good = dict(W=0x10000, numel=4096, dtype=0, dq_format=0, codes=0x10000, absmax=0x10000, qabs=0x10000,
                dq_scale=0x10000, dq_mean=0x10000)

    def call(n=2, wsb=512, ws_=ws, **bad):
        arr = (api.CQuantJob * 2)(api.CQuantJob(**good), api.CQuantJob(**dict(good, **bad)))
        return L.nf4_quantize_dq_batch(arr, n, ws_, wsb, None)
    assert L.nf4_quantize_dq_batch(None, 1, ws, 256, None) == 1
    assert call(ws_=None) == 1
    assert call(W=None) == 1                  # the second job is checked too
    assert call(n=0) == 2
    assert call(n=(1 << 20) + 1, wsb=1 << 40) == 2
    assert call(numel=0) == 2
    assert call(dtype=9) == 2
    assert call(dq_format=5) == 2
    assert call(absmax=0x10004) == 3
    assert call(ws_=P(0x20010)) == 3
    assert call(wsb=511) == 4
    assert api.workspace_bytes(api.OP_QUANTIZE_DQ_BATCH, 224) == 224 * 256
    assert api.workspace_bytes(api.OP_QUANTIZE_DQ_BATCH, 0) == 0


def test_quantize_dq_batch_wrapper_checks_outputs():
    """The Python wrapper rejects outputs of the wrong dtype, size or layout
    before the C call (CPU tensors: the checks come before the device check)."""
    import torch
    n = 4096
    nb = n // 64

    def job(**bad):
        t = dict(W=torch.zeros(n), codes=torch.zeros(n // 2, dtype=torch.uint8), absmax=torch.zeros(nb),
                 qabs=torch.zeros(nb, dtype=torch.int8), dq_scale=torch.zeros(1), dq_mean=torch.zeros(1), fmt="int8")
        t.update(bad)
        return (t["W"], t["codes"], t["absmax"], t["qabs"], t["dq_scale"], t["dq_mean"], t["fmt"])
    for bad, msg in ((dict(absmax=torch.zeros(nb, dtype=torch.float16)), "absmax must be"),
                     (dict(codes=torch.zeros(n // 2 - 1, dtype=torch.uint8)), "codes holds"),
                     (dict(qabs=torch.zeros(nb, dtype=torch.int16)), "qabs must be"),
                     (dict(dq_scale=torch.zeros(2, 2)[:, 0]), "dq_scale must be contiguous"),
                     (dict(dq_mean=torch.zeros(0)), "dq_mean holds"),
                     (dict(fmt="int4"), "unknown double-quantization format")):
        with pytest.raises(ValueError, match=msg):
            api.nf4_quantize_dq_batch([job(**bad), job()])
    with pytest.raises(ValueError, match="CUDA"):  # well-formed CPU tensors stop at the device check
        api.nf4_quantize_dq_batch([job()])


def test_dequant_argument_errors(L):
    out = A16
    assert L.nf4_dequant(None, out, None) == 1
    assert L.nf4_dequant(ctypes.byref(_w(codes=None)), out, None) == 1
    assert L.nf4_dequant(ctypes.byref(_w(absmax=None)), out, None) == 1         # no DQ and no absmax
    assert L.nf4_dequant(ctypes.byref(_w(absmax=None, qabs=A16)), out, None) == 1  # DQ without scale/mean
    assert L.nf4_dequant(ctypes.byref(_w(cols=96)), out, None) == 2
    assert L.nf4_dequant(ctypes.byref(_w(rows=0)), out, None) == 2
    assert L.nf4_dequant(ctypes.byref(_w(codes=P(0x10008))), out, None) == 3
    assert L.nf4_dequant(ctypes.byref(_w()), P(0x10002), None) == 3


def test_linear_argument_errors(L):
    w = _w(rows=128, cols=256)
    ws = P(0x40000)
    fwd = lambda **k: L.qlora_linear_fwd(ctypes.byref(k.get("w", w)), k.get("X", A16), k.get("n", 4),
                                         A16, A16, k.get("r", 16), 1.0, k.get("Y", A16), None,
                                         k.get("ws", ws), k.get("wsb", 1 << 30), None)
    assert fwd(X=None) == 1
    assert fwd(Y=None) == 1
    assert fwd(n=0) == 2
    assert fwd(r=12) == 2
    assert fwd(r=136) == 2
    assert fwd(w=_w(rows=100, cols=256)) == 2
    assert fwd(X=P(0x10008)) == 3
    assert fwd(ws=P(0x40010)) == 3
    need = api.workspace_bytes(api.OP_LINEAR_FWD, 128, 256, 4, 16)
    assert fwd(wsb=need - 1) == 4
    bwd = L.qlora_linear_bwd(ctypes.byref(w), A16, 4, A16, A16, 16, 1.0, None, None, A16, A16, A16, ws, 1 << 30,
                             None)
    assert bwd == 1
    need = api.workspace_bytes(api.OP_LINEAR_BWD, 128, 256, 4, 16)
    bwd = L.qlora_linear_bwd(ctypes.byref(w), A16, 4, A16, A16, 16, 1.0, A16, None, A16, A16, A16, ws, need - 1,
                             None)
    assert bwd == 4


def test_adamw_argument_errors(L):
    cfg = api.CAdamWConfig(1e-3, 0.9, 0.999, 1e-8, 0.0)
    c = ctypes.byref(cfg)
    assert L.qln_adamw_step(None, A16, A16, A16, None, 64, c, A16, 0, None) == 1
    assert L.qln_adamw_step(A16, A16, A16, A16, None, 64, None, A16, 0, None) == 1
    assert L.qln_adamw_step(A16, A16, A16, A16, None, 64, c, None, 0, None) == 1
    assert L.qln_adamw_step(A16, A16, A16, A16, None, 0, c, A16, 0, None) == 2
    assert L.qln_adamw_step(A4, A16, A16, A16, None, 64, c, A16, 0, None) == 3
    assert L.qln_adamw_step(A16, A16, A16, A4, None, 64, c, A16, 0, None) == 3
    assert L.qln_adamw_step(A16, A16, A16, A16, A4, 64, c, A16, 0, None) == 3


def test_quantize_ex_argument_errors(L):
    assert L.nf4_quantize_ex(None, api.DTYPE_BF16, 65, A16, A16, None) == 1
    assert L.nf4_quantize_ex(A16, api.DTYPE_BF16, 0, A16, A16, None) == 2
    assert L.nf4_quantize_ex(A16, 7, 64, A16, A16, None) == 2                    # unknown element type
    assert L.nf4_quantize_ex(A4, api.DTYPE_F16, 65, A16, A16, None) == 3
    assert L.nf4_quantize_ex(A16, api.DTYPE_F32, 65, A4, A16, None) == 3
    assert L.nf4_quantize_ex(A16, api.DTYPE_F32, 65, A16, P(0x10002), None) == 3


def test_double_quant_ex_argument_errors(L):
    ws = P(0x20000)
    need = api.workspace_bytes(api.OP_DOUBLE_QUANT, 100)
    assert L.nf4_double_quant_ex(None, 100, 0, A16, A16, A16, ws, need, None) == 1
    assert L.nf4_double_quant_ex(A16, 100, 2, A16, A16, A16, ws, need, None) == 2   # unknown 8-bit format
    assert L.nf4_double_quant_ex(A16, 0, 1, A16, A16, A16, ws, need, None) == 2
    assert L.nf4_double_quant_ex(A16, 100, 1, A16, A16, A16, P(0x20010), need, None) == 3
    assert L.nf4_double_quant_ex(A16, 100, 1, A16, A16, A16, ws, need - 1, None) == 4


def test_dequant_flat_and_format_argument_errors(L):
    out = A16
    w = _w()
    assert L.nf4_dequant_flat(None, 65, out, None) == 1
    assert L.nf4_dequant_flat(ctypes.byref(w), 0, out, None) == 2
    assert L.nf4_dequant_flat(ctypes.byref(w), 65, P(0x10002), None) == 3
    bad = _w()
    bad.dq_format = 9                                                            # neither INT8 nor E4M3
    assert L.nf4_dequant(ctypes.byref(bad), out, None) == 2
    assert L.nf4_dequant_flat(ctypes.byref(bad), 64, out, None) == 2


def test_noalloc_binding_rejects_wrong_dtypes_and_short_outputs():
    """The binding of the allocation-free double quantization checks what the
    library will write through raw pointers before calling it."""
    import pytest
    import torch
    from bit_nf4_quantized_07_b200 import api
    nb = 1000
    ok = dict(absmax=torch.zeros(nb), qabs=torch.zeros(nb, dtype=torch.int8),
              dq_scale=torch.zeros(4), dq_mean=torch.zeros(1))
    bad = [dict(ok, absmax=torch.zeros(nb, dtype=torch.float64)),
           dict(ok, qabs=torch.zeros(nb, dtype=torch.uint8)),
           dict(ok, qabs=torch.zeros(nb - 1, dtype=torch.int8)),
           dict(ok, dq_scale=torch.zeros(3)),
           dict(ok, dq_mean=torch.zeros(0)),
           dict(ok, dq_scale=torch.zeros(8)[::2])]
    for kw in bad:
        with pytest.raises(ValueError):
            api.nf4_double_quant_noalloc(**kw)
