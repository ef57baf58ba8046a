"""The allocation-free double quantization entry point.

nf4_double_quant_noalloc serves callers that cannot allocate device memory
where they quantize (a runtime that pre-reserves all device memory in its own
pool, a plugin handed tensors by a host framework): it keeps its scratch in a
fixed array inside the library instead of a caller workspace.  These tests
call it through the C ABI and require the same bits as nf4_double_quant, on
consecutive calls that share that array.  This file is collected last on
purpose (it also has to pass alone, in a fresh process).
"""
import ctypes

import numpy as np
import pytest

from bit_nf4_quantized_07_b200 import api, synthetic

MAX_BLOCKS = 1024 * 8192


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


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    import torch
    # First call spans four partial sums, the second only two: a stale partial
    # from the first call would change mu in the second.
    for seed, nb in ((41, 3 * 8192 + 5), (42, 8192 + 1), (43, 3670016)):
        a = torch.from_numpy(np.abs(synthetic.normal_f32(nb, 0.02, seed))).cuda()
        (rq, rs, rm), (q, s, m) = _reference_and_noalloc(a)
        assert torch.equal(q, rq), "qabs differs"
        assert torch.equal(s.view(torch.int32), rs.view(torch.int32)), "dq_scale differs"
        assert torch.equal(m.view(torch.int32), rm.view(torch.int32)), "dq_mean differs"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # Size checks happen before any device work, so fake addresses suffice.
    L = api.lib()
    fake = ctypes.c_void_p(0x10000)
    assert L.nf4_double_quant_noalloc(fake, MAX_BLOCKS + 1, fake, fake, fake, None) == 2
    assert L.nf4_double_quant_noalloc(fake, 0, fake, fake, fake, None) == 2
    assert L.nf4_double_quant_noalloc(None, 64, fake, fake, fake, None) == 1
