"""GPU parity of the codec kernels (quantize, double quantization, dequant)
against the CPU oracle: bit-exact codes, constants, mean and BF16 weights."""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_07_b200 import api, synthetic
from oracle import codec
from tests.oracle_ref import dev_bf16_bits

pytestmark = pytest.mark.gpu


def _gpu_codec(w: np.ndarray):
    W = torch.from_numpy(np.ascontiguousarray(w, np.float32)).cuda()
    rows, cols = w.reshape(-1, 64).shape[0], 64
    codes, absmax = api.nf4_quantize(W)
    qabs, scale, mu = api.nf4_double_quant(absmax)
    wq = api.NF4Weight(codes=codes, rows=rows, cols=cols, absmax=absmax, qabs=qabs, dq_scale=scale, dq_mean=mu)
    deq = api.nf4_dequant(wq)
    wplain = api.NF4Weight(codes=codes, rows=rows, cols=cols, absmax=absmax)
    deq_plain = api.nf4_dequant(wplain)
    torch.cuda.synchronize()
    return (codes.cpu().numpy(), absmax.cpu().numpy(), qabs.cpu().numpy(), scale.cpu().numpy(),
            mu.cpu().numpy()[0], dev_bf16_bits(deq).reshape(-1), dev_bf16_bits(deq_plain).reshape(-1))


def _check_all(w):
    n = w.size
    g = _gpu_codec(w)
    codes, absmax = codec.quantize(w)
    qabs, scale, mu = codec.double_quant(absmax)
    assert np.array_equal(g[1].view(np.uint32), absmax.view(np.uint32)), "absmax"
    assert np.array_equal(g[0], codes), f"codes: {np.sum(g[0] != codes)} bytes differ"
    assert np.float32(g[4]).view(np.uint32) == np.float32(mu).view(np.uint32), (g[4], mu)
    assert np.array_equal(g[3].view(np.uint32), scale.view(np.uint32)), "dq scale"
    assert np.array_equal(g[2], qabs), "dq codes"
    assert np.array_equal(g[5], codec.dequant(codes, n, qabs=qabs, scale=scale, mu=mu)), "dequant (DQ)"
    assert np.array_equal(g[6], codec.dequant(codes, n, absmax=absmax)), "dequant (plain)"


@pytest.mark.parametrize("shape,seed", [((512, 512), 1), ((1, 64), 2), ((3, 320), 3), ((77, 192), 4),
                                        ((1000, 192), 5), ((257, 256), 6), ((4096, 4096), 7)])
def test_codec_bit_exact(shape, seed):
    _check_all(synthetic.normal_f32(shape, 0.02, seed))


def test_codec_crafted_edge_blocks():
    cb = codec.cb32()
    blocks = []
    blocks.append(np.zeros(64, np.float32))                              # all zero
    b = np.zeros(64, np.float32); b[17] = -5.0; blocks.append(b)          # single nonzero
    blocks.append(np.full(64, -0.0, np.float32))                          # negative zeros
    b = np.zeros(64, np.float32); b[0], b[1] = 2.0, -2.0; blocks.append(b)  # +-absmax tie
    blocks.append(np.tile(np.r_[cb, cb[::-1]], 2).astype(np.float32) * np.float32(0.37))  # every code
    for k in range(15):                                                   # near/at every midpoint
        mid = (float(cb[k]) + float(cb[k + 1])) / 2
        m32 = np.float32(mid)
        b = np.full(64, m32, np.float32)
        b[0] = 1.0
        b[1:8] = np.nextafter(m32, np.float32(-2))
        b[8:16] = np.nextafter(m32, np.float32(2))
        b[16:24] = np.nextafter(np.nextafter(m32, np.float32(2)), np.float32(2))
        blocks.append(b)
    blocks.append(np.float32(1e-38) * np.linspace(-1, 1, 64, dtype=np.float32))   # subnormal-range block
    blocks.append(np.float32(3e38) * np.linspace(-1, 1, 64, dtype=np.float32))    # near fp32 max
    w = np.concatenate(blocks)
    _check_all(w)


def test_quantize_near_thresholds_with_inexact_reciprocals():
    """Blocks whose absmax is not a power of two, filled with fp32 values a few
    ulps either side of a * t_k for every threshold: the fast product w * (1/a)
    and the exact quotient w / a disagree by an ulp or two there, so every
    code checks the near-threshold fallback against the oracle's IEEE divide."""
    cb = codec.cb32().astype(np.float64)
    rng = np.random.Generator(np.random.PCG64(31))
    blocks = []
    for i in range(600):
        a = np.float32(rng.uniform(0.01, 100.0))
        b = np.empty(64, np.float32)
        b[0] = a if i % 2 == 0 else -a
        k = rng.integers(0, 15, 63)
        t = np.float32(a * (cb[k] + cb[k + 1]) / 2)
        steps = rng.integers(-3, 4, 63)
        for j in range(63):
            v = t[j]
            for _ in range(abs(int(steps[j]))):
                v = np.nextafter(v, np.float32(np.sign(steps[j]) * 1e9))
            b[1 + j] = v
        b[1:] = np.clip(b[1:], -a, a)
        blocks.append(b)
    _check_all(np.concatenate(blocks))


def test_quantize_16_byte_aligned_input():
    """W may be 16-byte but not 32-byte aligned (the wide-load path needs 32):
    same codes and constants as from an aligned copy, ragged last chunk."""
    w = synthetic.normal_f32((7 * 64 + 3 * 64,), 0.02, 41)
    buf = torch.zeros(w.size + 8, dtype=torch.float32, device="cuda")
    W = buf[4:4 + w.size]
    assert W.data_ptr() % 32 == 16
    W.copy_(torch.from_numpy(w))
    codes, absmax = api.nf4_quantize(W)
    torch.cuda.synchronize()
    c_ref, a_ref = codec.quantize(w)
    assert np.array_equal(codes.cpu().numpy(), c_ref)
    assert np.array_equal(absmax.cpu().numpy().view(np.uint32), a_ref.view(np.uint32))


def test_dq_degenerate_groups():
    w = np.tile(np.r_[np.float32(0.25), np.zeros(63, np.float32)], 600)   # all a_j equal -> b == 0
    _check_all(w)


def test_prefill_size_codec_bit_exact():
    cfg = synthetic.PREFILL
    _check_all(synthetic.weight_f32(cfg))


@pytest.mark.slow
def test_large_size_codec_sampled():
    """Full Large weight (28672 x 8192, 0.1 % x10 outliers) on the GPU; the
    oracle checks 8192 sampled blocks plus the first and last, the full absmax
    (NumPy max) and the full double quantization."""
    cfg = synthetic.LARGE
    w = synthetic.weight_f32(cfg)
    codes_g, absmax_g, qabs_g, scale_g, mu_g, deq_g, _ = _gpu_codec(w)
    wb = w.reshape(-1, 64)
    nb = wb.shape[0]
    assert np.array_equal(absmax_g, np.max(np.abs(wb), axis=1))
    qabs, scale, mu = codec.double_quant(absmax_g)
    assert np.float32(mu_g).view(np.uint32) == np.float32(mu).view(np.uint32)
    assert np.array_equal(qabs_g, qabs) and np.array_equal(scale_g.view(np.uint32), scale.view(np.uint32))
    rng = np.random.Generator(np.random.PCG64(99))
    idx = np.unique(np.r_[0, nb - 1, rng.integers(0, nb, 8192)])
    codes_s, _ = codec.quantize(wb[idx])
    assert np.array_equal(codes_g.reshape(nb, 32)[idx], codes_s.reshape(-1, 32))
    # dequant of the sampled blocks with the full-tensor DQ constants
    deq = deq_g.reshape(nb, 64)[idx]
    for k, j in enumerate(idx[:512]):
        ah = codec.dq_restore(qabs[j:j + 1], scale[j // 256:j // 256 + 1], mu)[0]
        ref = codec.dequant(codes_s.reshape(-1, 32)[k], 64, absmax=np.array([ah], np.float32))
        assert np.array_equal(deq[k], ref)


RAGGED = [1, 2, 7, 63, 64, 65, 130, 1000, 4096 + 37, (1 << 20) + 5, 3 * 1024 + 999]


def _to_kind(w32: np.ndarray, kind: str):
    """fp32 values -> (device tensor of that dtype, oracle input bits or values)."""
    t = torch.from_numpy(w32)
    if kind == "f32":
        return t.cuda(), w32
    dt = torch.bfloat16 if kind == "bf16" else torch.float16
    d = t.to(dt)
    return d.cuda(), d.view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("kind", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("n", RAGGED)
def test_quantize_any_dtype_and_numel_bit_exact(kind, n):
    """nf4_quantize_ex (and nf4_dequant_flat) against the oracle for 16-bit and
    fp32 weights of any numel: codes, absmax, DQ and BF16 bits exact, and no
    byte written past ceil(n/2) codes / n outputs."""
    w32 = synthetic.normal_f32((n,), 0.02, 700 + n)
    W, ref_in = _to_kind(w32, kind)
    guard = 37
    codes = torch.full(((n + 1) // 2 + guard,), 0xAB, dtype=torch.uint8, device="cuda")
    absmax = torch.full(((n + 63) // 64 + 1,), -1.0, dtype=torch.float32, device="cuda")
    api.nf4_quantize(W, codes=codes[:(n + 1) // 2], absmax=absmax[:(n + 63) // 64])
    c_ref, a_ref = codec.quantize(ref_in) if kind == "f32" else codec.quantize16(ref_in, kind)
    torch.cuda.synchronize()
    cg = codes.cpu().numpy()
    ag = absmax.cpu().numpy()
    assert np.array_equal(cg[:(n + 1) // 2], c_ref), f"codes: {np.sum(cg[:(n + 1) // 2] != c_ref)} differ"
    assert np.all(cg[(n + 1) // 2:] == 0xAB), "wrote past the codes"
    assert np.array_equal(ag[:-1].view(np.uint32), a_ref.view(np.uint32)), "absmax"
    assert ag[-1] == -1.0, "wrote past absmax"
    # DQ + flat dequant of the ragged weight
    am = absmax[:(n + 63) // 64]
    qabs, scale, mu = api.nf4_double_quant(am)
    q_ref, s_ref, mu_ref = codec.double_quant(a_ref)
    wq = api.NF4Weight(codes=codes[:(n + 1) // 2], rows=1, cols=n, absmax=am, qabs=qabs, dq_scale=scale, dq_mean=mu)
    out = torch.full((n + 24,), 0x7FC1, dtype=torch.int16, device="cuda")
    api.nf4_dequant_flat(wq, n, out=out[:n].view(torch.bfloat16))
    torch.cuda.synchronize()
    assert np.array_equal(qabs.cpu().numpy(), q_ref) and np.float32(mu.item()) == np.float32(mu_ref)
    og = out.cpu().numpy().view(np.uint16)
    assert np.array_equal(og[:n], codec.dequant(c_ref, n, qabs=q_ref, scale=s_ref, mu=mu_ref)), "dequant"
    assert np.all(og[n:] == 0x7FC1), "wrote past the dequant output"


def test_quantize16_matches_fp32_path_on_prefill_weight():
    """bf16 weights of the prefill layer: the 16-bit path gives the bytes the
    fp32 path gives for the widened values."""
    cfg = synthetic.PREFILL
    w = torch.from_numpy(synthetic.weight_f32(cfg)).cuda().to(torch.bfloat16)
    c16, a16 = api.nf4_quantize(w)
    c32, a32 = api.nf4_quantize(w.float())
    torch.cuda.synchronize()
    assert torch.equal(c16, c32) and torch.equal(a16, a32)


@pytest.mark.parametrize("shape,seed", [((512, 512), 51), ((3, 320), 52), ((1000, 192), 53), ((11008, 4096), 54)])
def test_e4m3_double_quant_and_dequant_bit_exact(shape, seed):
    """The "8-bit floats" DQ format: E4M3 codes, group scales, mu and the BF16
    dequant (tiled and flat) bit-exact against the oracle."""
    w = synthetic.normal_f32(shape, 0.02, seed)
    W = torch.from_numpy(w).cuda()
    codes, absmax = api.nf4_quantize(W)
    q, b, mu = api.nf4_double_quant(absmax, fmt="e4m3")
    rows, cols = w.reshape(-1, 64).shape[0], 64
    wq = api.NF4Weight(codes=codes, rows=rows, cols=cols, absmax=absmax, qabs=q, dq_scale=b, dq_mean=mu,
                       dq_format="e4m3")
    deq = api.nf4_dequant(wq)
    flat = api.nf4_dequant_flat(wq, w.size)
    torch.cuda.synchronize()
    c_ref, a_ref = codec.quantize(w)
    q_ref, b_ref, mu_ref = codec.double_quant(a_ref, fmt="e4m3")
    assert np.array_equal(q.cpu().numpy(), q_ref), f"{np.sum(q.cpu().numpy() != q_ref)} E4M3 codes differ"
    assert np.array_equal(b.cpu().numpy().view(np.uint32), b_ref.view(np.uint32))
    assert np.float32(mu.item()).view(np.uint32) == np.float32(mu_ref).view(np.uint32)
    ref = codec.dequant(c_ref, w.size, qabs=q_ref, scale=b_ref, mu=mu_ref, fmt="e4m3")
    assert np.array_equal(dev_bf16_bits(deq).reshape(-1), ref)
    assert np.array_equal(dev_bf16_bits(flat).reshape(-1), ref)


@pytest.mark.parametrize("fmt", ["int8", "e4m3"])
def test_single_launch_dq_repeats_replays_and_leaves_header_zeroed(fmt):
    """The single-launch double quantization (grid barrier on counters in the
    workspace header): back-to-back calls and CUDA graph replays on one
    workspace give the oracle's bits, and every call leaves the header at zero."""
    w = synthetic.normal_f32((11008 // 4, 4096), 0.02, 61)
    codes, absmax = api.nf4_quantize(torch.from_numpy(w).cuda())
    nb = absmax.numel()
    ws = api.alloc_workspace(api.workspace_bytes(api.OP_DOUBLE_QUANT, nb))
    _, a_ref = codec.quantize(w)
    q_ref, b_ref, mu_ref = codec.double_quant(a_ref, fmt=fmt)
    q, b, mu = api.nf4_double_quant(absmax, ws=ws, fmt=fmt)
    for _ in range(3):
        q2, b2, mu2 = api.nf4_double_quant(absmax, ws=ws, fmt=fmt)
        assert torch.equal(q, q2) and torch.equal(b, b2) and torch.equal(mu, mu2)
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy().view(np.uint8), q_ref.view(np.uint8))
    assert np.array_equal(b.cpu().numpy().view(np.uint32), b_ref.view(np.uint32))
    assert np.float32(mu.item()).view(np.uint32) == np.float32(mu_ref).view(np.uint32)
    assert int(ws[:256].view(torch.int32).abs().sum().item()) == 0
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        api.nf4_double_quant(absmax, q, b, mu, ws=ws, fmt=fmt)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(3):
            api.nf4_double_quant(absmax, q, b, mu, ws=ws, fmt=fmt)
    q.zero_()
    for _ in range(4):
        graph.replay()
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy().view(np.uint8), q_ref.view(np.uint8))
    assert int(ws[:256].view(torch.int32).abs().sum().item()) == 0


def test_single_launch_dq_barrier_runs_out_and_reports_timeout():
    """Failure detection without a GPU fault: an arrival counter that can
    never reach the grid size makes every CTA's bounded barrier wait (2 s) run
    out; the kernel records QLN_ERR_TIMEOUT and finishes.  With the header
    zeroed again the next call is exact."""
    import time
    w = synthetic.normal_f32((1024, 4096), 0.02, 62)
    codes, absmax = api.nf4_quantize(torch.from_numpy(w).cuda())
    nb = absmax.numel()
    ws = api.alloc_workspace(api.workspace_bytes(api.OP_DOUBLE_QUANT, nb))
    ws[64:68].view(torch.int32).fill_(-(1 << 30))  # the barrier's arrival counter
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    api.nf4_double_quant(absmax, ws=ws)
    torch.cuda.synchronize()
    assert 1.0 < time.perf_counter() - t0 < 60.0
    assert api.device_status(ws) == 7, "QLN_ERR_TIMEOUT expected"
    ws[:256].zero_()
    q, b, mu = api.nf4_double_quant(absmax, ws=ws)
    torch.cuda.synchronize()
    assert api.device_status(ws) == 0
    q_ref, b_ref, mu_ref = codec.double_quant(codec.quantize(w)[1])
    assert np.array_equal(q.cpu().numpy(), q_ref) and np.float32(mu.item()) == np.float32(mu_ref)
