"""The allocation-free double quantization entry point.

nf4_double_quant_noalloc serves callers that cannot allocate device memory
where they quantize (a runtime that pre-reserves all device memory in its own
pool, a plugin handed tensors by a host framework): it keeps its scratch in a
fixed array inside the library instead of a caller workspace.  These tests
call it through the C ABI and require the same bits as nf4_double_quant and
as the oracle, on consecutive calls that share that array.  This file is collected last on
purpose (it also has to pass alone, in a fresh process).
"""
import ctypes

import numpy as np
import pytest

from bit_nf4_quantized_07_b200 import api, synthetic
from oracle import codec as ocodec

MAX_BLOCKS = 1 << 25


def _reference_and_noalloc(absmax):
    import torch
    nb = absmax.numel()
    ref = api.nf4_double_quant(absmax)
    qabs = torch.full((nb,), 77, dtype=torch.int8, device="cuda")
    scale = torch.full(((nb + 255) // 256,), 1.5, dtype=torch.float32, device="cuda")
    mean = torch.full((1,), -3.0, dtype=torch.float32, device="cuda")
    L = api.lib()
    st = L.nf4_double_quant_noalloc(ctypes.c_void_p(absmax.data_ptr()), nb, ctypes.c_void_p(qabs.data_ptr()),
                                     ctypes.c_void_p(scale.data_ptr()), ctypes.c_void_p(mean.data_ptr()),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, api.status_str(st)
    torch.cuda.synchronize()
    return ref, (qabs, scale, mean)


def _spread_constants(nb, seed):
    """Constants whose magnitudes span many powers of two (subnormals to 1e30),
    so the exact sum's runs fall on different limbs within one warp."""
    rng = np.random.default_rng(seed)
    a = (rng.random(nb) * 10.0 ** rng.integers(-44, 31, nb)).astype(np.float32)
    a[rng.integers(0, nb, 16)] = np.float32(1.4e-45)
    return a


@pytest.mark.gpu
@pytest.mark.parametrize("case", ["multi", "single", "prefill", "2^23", "spread"])
def test_noalloc_matches_workspace_entry_point_and_oracle(case):
    import torch
    # Runs in this order in one process: every call starts from the scratch the
    # previous one left behind, so a sum not put back to zero changes mu.
    seed, nb = {"multi": (41, 3 * 8192 + 5), "single": (42, 8192 + 1), "prefill": (43, 3670016),
                "2^23": (44, 8388608), "spread": (45, 70001)}[case]
    a_np = _spread_constants(nb, seed) if case == "spread" else np.abs(synthetic.normal_f32(nb, 0.02, seed))
    a = torch.from_numpy(a_np).cuda()
    (rq, rs, rm), (q, s, m) = _reference_and_noalloc(a)
    assert torch.equal(q, rq), "qabs differs from nf4_double_quant"
    assert torch.equal(s.view(torch.int32), rs.view(torch.int32)), "dq_scale differs from nf4_double_quant"
    assert torch.equal(m.view(torch.int32), rm.view(torch.int32)), "dq_mean differs from nf4_double_quant"
    oq, os_, om = ocodec.double_quant(a_np)
    assert np.float32(om).view(np.uint32) == m.cpu().numpy().view(np.uint32)[0], "dq_mean differs from the oracle"
    assert np.array_equal(s.cpu().numpy().view(np.uint32), np.asarray(os_, np.float32).view(np.uint32)), \
        "dq_scale differs from the oracle"
    assert np.array_equal(q.cpu().numpy(), np.asarray(oq, np.int8)), "qabs differs from the oracle"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # Size checks happen before any device work, so fake addresses suffice.
    L = api.lib()
    fake = ctypes.c_void_p(0x10000)
    assert L.nf4_double_quant_noalloc(fake, MAX_BLOCKS + 1, fake, fake, fake, None) == 2
    assert L.nf4_double_quant_noalloc(fake, 0, fake, fake, fake, None) == 2
    assert L.nf4_double_quant_noalloc(None, 64, fake, fake, fake, None) == 1
