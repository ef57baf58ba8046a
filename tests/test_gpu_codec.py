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


def _scratch_at_rest(ws):
    """The DQ scratch between calls: status 0, arrival counter 0 and the bank of
    limbs the next call sums into (bank gen % 2) all zero."""
    w = ws[:256].view(torch.int32).cpu().numpy()
    gen = int(w[4])                                   # generation word at byte 16
    bank = w[16:36] if gen % 2 == 0 else w[40:60]     # banks at bytes 64 and 160, 80 bytes each
    return w[0] == 0 and w[8] == 0 and not bank.any()


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
    """The single-launch double quantization (grid barrier on counters and the
    exact sum in the workspace header): back-to-back calls, a call on another
    stream and CUDA graph replays on one workspace give the oracle's bits, and
    every call leaves the scratch ready for the next one."""
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
    assert _scratch_at_rest(ws)
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
    assert _scratch_at_rest(ws)


def test_single_launch_dq_barrier_runs_out_and_reports_timeout():
    """Failure detection without a GPU fault: an arrival counter that can
    never count the last CTA in leaves the generation where it is, so every
    CTA's bounded barrier wait (2 s) runs out; the kernel records
    QLN_ERR_TIMEOUT and finishes.  With the header zeroed again the next call
    is exact."""
    import time
    w = synthetic.normal_f32((1024, 4096), 0.02, 62)
    codes, absmax = api.nf4_quantize(torch.from_numpy(w).cuda())
    nb = absmax.numel()
    ws = api.alloc_workspace(api.workspace_bytes(api.OP_DOUBLE_QUANT, nb))
    ws[32:36].view(torch.int32).fill_(-(1 << 30))  # the barrier's arrival counter: no CTA is ever last
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


def _spread_constants(nb, seed):
    """Block constants spanning subnormals to 1e30 (and some negative ones,
    which the entry point accepts): the exact sum's runs fall on different
    limbs inside one warp and the sum changes sign along the way."""
    rng = np.random.default_rng(seed)
    a = (rng.random(nb) * 10.0 ** rng.integers(-44, 31, nb)).astype(np.float32)
    a[rng.integers(0, nb, max(1, nb // 50))] *= -1
    a[rng.integers(0, nb, 8)] = np.float32(1.4e-45)
    return a


@pytest.mark.parametrize("nb", [1, 255, 257, 70001, 2000003, 3670016, 6000001])
@pytest.mark.parametrize("kind", ["normal", "spread"])
def test_double_quant_every_launch_shape_matches_oracle(nb, kind):
    """Direct double quantization of block constants against the oracle, at
    sizes that take each launch shape on a 148-SM B200: one group per warp
    (nb <= 1.8 M), two (<= 2.4 M), four (<= 4.8 M) in the single cooperative
    launch, and the two-launch path beyond.  mu must be the oracle's bits."""
    a = (np.abs(synthetic.normal_f32(nb, 0.02, 70 + nb % 97)) if kind == "normal"
         else _spread_constants(nb, 71 + nb % 89))
    q, b, mu = api.nf4_double_quant(torch.from_numpy(a).cuda())
    torch.cuda.synchronize()
    q_ref, b_ref, mu_ref = codec.double_quant(a)
    assert np.float32(mu.item()).view(np.uint32) == np.float32(mu_ref).view(np.uint32), (mu.item(), mu_ref)
    assert np.array_equal(b.cpu().numpy().view(np.uint32), b_ref.view(np.uint32)), "dq scale"
    assert np.array_equal(q.cpu().numpy(), q_ref), f"{np.sum(q.cpu().numpy() != q_ref)} dq codes differ"


@pytest.mark.parametrize("numel,dtype,fmt,seed", [
    (64, torch.float32, "int8", 80), (4096 * 4096, torch.float32, "int8", 81), (1000 * 192 + 37, torch.float32, "int8", 82),
    (11008 * 512, torch.bfloat16, "int8", 83), (333333, torch.float16, "e4m3", 84), (5 * 16384 + 1, torch.bfloat16, "e4m3", 85)])
def test_quantize_dq_one_call_matches_oracle(numel, dtype, fmt, seed):
    """nf4_quantize_dq (quantize with the exact sum formed on the way, then the
    group quantization) against the oracle's quantize + double_quant of the
    same weights, ragged tails and every input dtype included; repeated calls
    on one workspace give the same bits and leave its scratch ready for the
    next call."""
    w = synthetic.normal_f32(numel, 0.02, seed)
    Wc = torch.from_numpy(w).to(dtype)          # rounded to the input dtype on the host
    w_exact = Wc.float().numpy()                # the values the kernel sees (widening is exact)
    Wd = Wc.cuda()
    ws = api.alloc_workspace(api.workspace_bytes(api.OP_DOUBLE_QUANT, (numel + 63) // 64))
    out = api.nf4_quantize_dq(Wd, ws=ws, fmt=fmt)
    again = api.nf4_quantize_dq(Wd, ws=ws, fmt=fmt)
    torch.cuda.synchronize()
    codes, absmax, q, b, mu = [t.cpu().numpy() for t in out]
    c_ref, a_ref = codec.quantize(w_exact)
    q_ref, b_ref, mu_ref = codec.double_quant(a_ref, fmt=fmt)
    assert np.array_equal(codes, c_ref), f"{np.sum(codes != c_ref)} code bytes differ"
    assert np.array_equal(absmax.view(np.uint32), a_ref.view(np.uint32))
    assert np.float32(mu[0]).view(np.uint32) == np.float32(mu_ref).view(np.uint32), (mu[0], mu_ref)
    assert np.array_equal(b.view(np.uint32), b_ref.view(np.uint32)), "dq scale"
    assert np.array_equal(q.view(np.uint8), q_ref.view(np.uint8)), "dq codes"
    for x, y in zip(out, again):
        assert torch.equal(x, y)
    assert api.device_status(ws) == 0
    assert _scratch_at_rest(ws)


def test_single_launch_dqs_near_the_size_limit_on_two_unordered_streams():
    """Two single-launch double quantizations, each with a grid of about 3/4 of
    what the device holds at once (four groups per warp, 4.5 M constants), on
    two streams with no order between them.  The cooperative launch keeps each
    grid's CTAs resident together, so both grid barriers complete: status
    QLN_OK and the oracle's bits for both."""
    nb = 4_500_000
    a_np = [np.abs(synthetic.normal_f32(nb, 0.02, 90 + k)) for k in range(2)]
    a = [torch.from_numpy(x).cuda() for x in a_np]
    ws = [api.alloc_workspace(api.workspace_bytes(api.OP_DOUBLE_QUANT, nb)) for _ in range(2)]
    outs = [(torch.empty(nb, dtype=torch.int8, device="cuda"), torch.empty((nb + 255) // 256, device="cuda"),
             torch.empty(1, device="cuda")) for _ in range(2)]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    torch.cuda.synchronize()
    for rep in range(3):
        for k in range(2):
            with torch.cuda.stream(streams[k]):
                api.nf4_double_quant(a[k], *outs[k], ws=ws[k])
    torch.cuda.synchronize()
    for k in range(2):
        assert api.device_status(ws[k]) == 0, api.status_str(api.device_status(ws[k]))
        q_ref, b_ref, mu_ref = codec.double_quant(a_np[k])
        q, b, mu = (t.cpu().numpy() for t in outs[k])
        assert np.float32(mu[0]).view(np.uint32) == np.float32(mu_ref).view(np.uint32)
        assert np.array_equal(b.view(np.uint32), b_ref.view(np.uint32))
        assert np.array_equal(q, q_ref)
        assert _scratch_at_rest(ws[k])


def test_quantize_dq_constants_spanning_many_binades():
    """nf4_quantize_dq on weights whose blocks are scaled by 10^-30 .. 10^30:
    the block constants a warp sums fall on different limbs of the exact sum,
    which takes the lane-by-lane path; mu, scales and codes still match the
    oracle bit for bit."""
    rng = np.random.default_rng(95)
    nblk = 300_001
    w = (rng.standard_normal((nblk, 64)) * 10.0 ** rng.integers(-30, 31, (nblk, 1))).astype(np.float32)
    Wd = torch.from_numpy(w).cuda()
    out = api.nf4_quantize_dq(Wd)
    torch.cuda.synchronize()
    codes, absmax, q, b, mu = [t.cpu().numpy() for t in out]
    c_ref, a_ref = codec.quantize(w)
    q_ref, b_ref, mu_ref = codec.double_quant(a_ref)
    assert np.array_equal(absmax.view(np.uint32), a_ref.view(np.uint32))
    assert np.array_equal(codes, c_ref)
    assert np.float32(mu[0]).view(np.uint32) == np.float32(mu_ref).view(np.uint32), (mu[0], mu_ref)
    assert np.array_equal(b.view(np.uint32), b_ref.view(np.uint32))
    assert np.array_equal(q, q_ref)


def test_int8_dq_rint_ties_worked_by_hand():
    """The hand-worked tie group (mu = 200, b = 1, quotients +-{127, 2.5, 3.5,
    0.5, 1.5}) through the device double quantization, alone and as part of a
    larger array whose extra constants are all equal to mu."""
    d = np.array([127, -127, 2.5, -2.5, 3.5, -3.5, 0.5, -0.5, 1.5, -1.5], np.float64)
    a = (200.0 + d).astype(np.float32)
    for arr in (a, np.concatenate([a, np.full(1000, 200.0, np.float32)])):
        q, b, mu = api.nf4_double_quant(torch.from_numpy(arr).cuda())
        torch.cuda.synchronize()
        assert mu.item() == 200.0 and b[0].item() == 1.0
        assert q[:10].cpu().tolist() == [127, -127, 2, -2, 4, -4, 0, 0, 2, -2]


@pytest.mark.parametrize("n", [1, 128])
def test_dq_restore_order_worked_by_hand(n):
    """ahat = fp32(mu + fp32(b rhat)) with b = 1 + 2^-23, rhat = 3, mu = -3 is
    2^-21 (an FMA would give 3 2^-23), worked by hand.  A 128 x 64 weight whose
    codes all hold the book's 1.0: nf4_dequant gives bf16(2^-21) everywhere,
    and the fused forward with one-hot token rows and B = 0 returns that
    weight, through the decode-sized kernel (n = 1) and the tensor-core GEMM
    (n = 128)."""
    rows, cols = 128, 64
    nb = rows * cols // 64
    codes = torch.full((rows * cols // 2,), 0xFF, dtype=torch.uint8, device="cuda")
    qabs = torch.full((nb,), 3, dtype=torch.int8, device="cuda")
    scale = torch.tensor([1.0 + 2.0 ** -23], dtype=torch.float32, device="cuda")
    mu = torch.tensor([-3.0], dtype=torch.float32, device="cuda")
    absmax = torch.zeros(nb, dtype=torch.float32, device="cuda")
    wq = api.NF4Weight(codes=codes, rows=rows, cols=cols, absmax=absmax, qabs=qabs, dq_scale=scale, dq_mean=mu)
    deq = api.nf4_dequant(wq)
    X = torch.zeros(n, cols, dtype=torch.bfloat16, device="cuda")
    X[torch.arange(n), torch.arange(n) % cols] = 1.0
    A = torch.zeros(16, cols, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(rows, 16, dtype=torch.bfloat16, device="cuda")
    Y, _ = api.qlora_linear_fwd(wq, X, A, B, 1.0)
    torch.cuda.synchronize()
    assert np.all(dev_bf16_bits(deq) == 0x3500)
    assert np.all(dev_bf16_bits(Y) == 0x3500)


BATCH_SHAPES = [(64 * 1000 + 37, torch.float32, "int8"), (4096 * 1024, torch.bfloat16, "int8"),
                (333_333, torch.float16, "e4m3"), (64, torch.float32, "int8"), (11008 * 256, torch.float32, "int8")]


@pytest.mark.parametrize("njobs", [1, 2, 3, 5])
def test_quantize_dq_batch_matches_oracle_per_job(njobs):
    """nf4_quantize_dq_batch: every job's codes, constants, DQ codes, scales and
    mu equal the oracle's quantize + double_quant of that job (the quantize
    launches back to back, then the sums and groups of all jobs in the tail
    launches).  A second call on the same workspace gives the same bits, and
    the scratch of every job is ready for the next call."""
    shapes = [BATCH_SHAPES[k % len(BATCH_SHAPES)] for k in range(njobs)]
    jobs, host = [], []
    for k, (numel, dtype, fmt) in enumerate(shapes):
        w = synthetic.normal_f32(numel, 0.02 * (k + 1), 120 + k)
        Wc = torch.from_numpy(w).to(dtype)
        host.append((Wc.float().numpy(), fmt))
        nb = (numel + 63) // 64
        jobs.append((Wc.cuda(), torch.empty((numel + 1) // 2, dtype=torch.uint8, device="cuda"),
                     torch.empty(nb, device="cuda"),
                     torch.empty(nb, dtype=torch.int8 if fmt == "int8" else torch.uint8, device="cuda"),
                     torch.empty((nb + 255) // 256, device="cuda"), torch.empty(1, device="cuda"), fmt))
    ws = api.alloc_workspace(api.workspace_bytes(api.OP_QUANTIZE_DQ_BATCH, njobs))
    api.nf4_quantize_dq_batch(jobs, ws=ws)
    torch.cuda.synchronize()
    first = [[t.clone() for t in j[1:6]] for j in jobs]
    api.nf4_quantize_dq_batch(jobs, ws=ws)
    torch.cuda.synchronize()
    assert api.device_status(ws) == 0
    for k, ((w_exact, fmt), j) in enumerate(zip(host, jobs)):
        for a, b in zip(first[k], j[1:6]):
            assert torch.equal(a, b), f"job {k}: second call differs"
        assert _scratch_at_rest(ws[256 * k:256 * (k + 1)])
        codes, absmax, q, b, mu = [t.cpu().numpy() for t in j[1:6]]
        c_ref, a_ref = codec.quantize(w_exact)
        q_ref, b_ref, mu_ref = codec.double_quant(a_ref, fmt=fmt)
        assert np.array_equal(codes, c_ref), f"job {k}: codes"
        assert np.array_equal(absmax.view(np.uint32), a_ref.view(np.uint32)), f"job {k}: absmax"
        assert np.float32(mu[0]).view(np.uint32) == np.float32(mu_ref).view(np.uint32), f"job {k}: mu"
        assert np.array_equal(b.view(np.uint32), b_ref.view(np.uint32)), f"job {k}: dq scale"
        assert np.array_equal(q.view(np.uint8), q_ref.view(np.uint8)), f"job {k}: dq codes"


def test_quantize_dq_batch_with_shared_outputs_runs_in_order():
    """Jobs whose outputs overlap (the second weight written into the first
    one's buffers) take the ordered schedule: the result is that of the second
    job, as with separate nf4_quantize_dq calls in order."""
    numel = 4096 * 256
    nb = numel // 64
    wa = synthetic.normal_f32(numel, 0.02, 131)
    wb = synthetic.normal_f32(numel, 0.05, 132)
    outs = (torch.empty(numel // 2, dtype=torch.uint8, device="cuda"), torch.empty(nb, device="cuda"),
            torch.empty(nb, dtype=torch.int8, device="cuda"), torch.empty(nb // 256, device="cuda"),
            torch.empty(1, device="cuda"))
    jobs = [(torch.from_numpy(wa).cuda(), *outs, "int8"), (torch.from_numpy(wb).cuda(), *outs, "int8")]
    api.nf4_quantize_dq_batch(jobs)
    torch.cuda.synchronize()
    codes, absmax, q, b, mu = [t.cpu().numpy() for t in outs]
    c_ref, a_ref = codec.quantize(wb)
    q_ref, b_ref, mu_ref = codec.double_quant(a_ref)
    assert np.array_equal(codes, c_ref) and np.array_equal(absmax.view(np.uint32), a_ref.view(np.uint32))
    assert np.float32(mu[0]).view(np.uint32) == np.float32(mu_ref).view(np.uint32)
    assert np.array_equal(b.view(np.uint32), b_ref.view(np.uint32)) and np.array_equal(q, q_ref)


def test_quantize_dq_batch_long_chain_and_shared_input():
    """A batch of 24 small weights of assorted sizes (a long quantize chain,
    then one tail launch pair whose CTA ranges cover jobs of very different
    sizes), two of them quantizing the same input tensor (read-only overlap
    keeps the early-start schedule): every job equals the oracle."""
    rng = np.random.default_rng(140)
    jobs, host = [], []
    shared = None
    for k in range(24):
        numel = int(rng.integers(1, 40)) * 4096 + int(rng.integers(0, 64))
        if k == 7:
            Wd, w = shared
        else:
            w = synthetic.normal_f32(numel, float(rng.uniform(0.005, 0.05)), 150 + k)
            Wd = torch.from_numpy(w).cuda()
            if k == 3:
                shared = (Wd, w)
        numel = w.size
        nb = (numel + 63) // 64
        host.append(w)
        jobs.append((Wd, torch.empty((numel + 1) // 2, dtype=torch.uint8, device="cuda"),
                     torch.empty(nb, device="cuda"), torch.empty(nb, dtype=torch.int8, device="cuda"),
                     torch.empty((nb + 255) // 256, device="cuda"), torch.empty(1, device="cuda"), "int8"))
    api.nf4_quantize_dq_batch(jobs)
    torch.cuda.synchronize()
    for k, (w, j) in enumerate(zip(host, jobs)):
        codes, absmax, q, b, mu = [t.cpu().numpy() for t in j[1:6]]
        c_ref, a_ref = codec.quantize(w)
        q_ref, b_ref, mu_ref = codec.double_quant(a_ref)
        assert np.array_equal(codes, c_ref), f"job {k}: codes"
        assert np.float32(mu[0]).view(np.uint32) == np.float32(mu_ref).view(np.uint32), f"job {k}: mu"
        assert np.array_equal(b.view(np.uint32), b_ref.view(np.uint32)), f"job {k}: dq scale"
        assert np.array_equal(q, q_ref), f"job {k}: dq codes"


@pytest.mark.gpu
def test_quantize_dq_batch_chained_through_an_earlier_output():
    """Three jobs where the third quantizes the first one's block constants
    (its weights are job 0's absmax buffer): the buffers overlap, so the
    ordered schedule runs, and the result is that of separate calls in order."""
    n0, n1 = 256 * 1024, 64 * 4096 + 40
    w0 = synthetic.normal_f32(n0, 0.02, 160)
    w1 = synthetic.normal_f32(n1, 0.03, 161)

    def outs(numel):
        nb = (numel + 63) // 64
        return (torch.empty((numel + 1) // 2, dtype=torch.uint8, device="cuda"), torch.empty(nb, device="cuda"),
                torch.empty(nb, dtype=torch.int8, device="cuda"), torch.empty((nb + 255) // 256, device="cuda"),
                torch.empty(1, device="cuda"))
    o0, o1 = outs(n0), outs(n1)
    o2 = outs(n0 // 64)
    jobs = [(torch.from_numpy(w0).cuda(), *o0, "int8"), (torch.from_numpy(w1).cuda(), *o1, "int8"),
            (o0[1], *o2, "int8")]
    api.nf4_quantize_dq_batch(jobs)
    torch.cuda.synchronize()
    c0, a0 = codec.quantize(w0)
    c1, a1 = codec.quantize(w1)
    c2, a2 = codec.quantize(np.asarray(a0, np.float32))
    for k, (o, (c_ref, a_ref)) in enumerate(zip((o0, o1, o2), ((c0, a0), (c1, a1), (c2, a2)))):
        codes, absmax, q, b, mu = [t.cpu().numpy() for t in o]
        q_ref, b_ref, mu_ref = codec.double_quant(a_ref)
        assert np.array_equal(codes, c_ref), f"job {k}: codes"
        assert np.array_equal(absmax.view(np.uint32), np.asarray(a_ref, np.float32).view(np.uint32)), f"job {k}: absmax"
        assert np.float32(mu[0]).view(np.uint32) == np.float32(mu_ref).view(np.uint32), f"job {k}: mu"
        assert np.array_equal(b.view(np.uint32), np.asarray(b_ref, np.float32).view(np.uint32)), f"job {k}: scales"
        assert np.array_equal(q, np.asarray(q_ref, np.int8)), f"job {k}: qabs"


@pytest.mark.gpu
def test_quantize_dq_batch_spanning_several_tail_launches():
    """131 weights, from one element to a few groups of constants: the double
    quantization takes two tail launch pairs (128 jobs per launch), and jobs
    of a single CTA sit next to jobs of several.  Every job equals the oracle,
    also after a second call on the same workspace."""
    rng = np.random.default_rng(141)
    jobs, host = [], []
    for k in range(131):
        numel = [1, 63, 64, 65][k] if k < 4 else int(rng.integers(1, 9)) * 16384 + int(rng.integers(0, 130))
        w = synthetic.normal_f32(numel, float(rng.uniform(0.005, 0.05)), 300 + k)
        nb = (numel + 63) // 64
        host.append(w)
        jobs.append((torch.from_numpy(w).cuda(), torch.empty((numel + 1) // 2, dtype=torch.uint8, device="cuda"),
                     torch.empty(nb, device="cuda"), torch.empty(nb, dtype=torch.int8, device="cuda"),
                     torch.empty((nb + 255) // 256, device="cuda"), torch.empty(1, device="cuda"), "int8"))
    refs = []
    for w in host:
        c_ref, a_ref = codec.quantize(w)
        refs.append((c_ref, a_ref) + tuple(codec.double_quant(a_ref)))
    ws = api.alloc_workspace(api.workspace_bytes(api.OP_QUANTIZE_DQ_BATCH, len(jobs)))
    for call in range(2):
        for j in jobs:
            for t in j[1:6]:
                t.fill_(0)
        api.nf4_quantize_dq_batch(jobs, ws=ws)
        torch.cuda.synchronize()
        assert api.device_status(ws) == 0
        for k, (ref, j) in enumerate(zip(refs, jobs)):
            codes, absmax, q, b, mu = [t.cpu().numpy() for t in j[1:6]]
            c_ref, a_ref, q_ref, b_ref, mu_ref = ref
            assert np.array_equal(codes, c_ref), f"call {call}, job {k}: codes"
            assert np.array_equal(absmax.view(np.uint32), a_ref.view(np.uint32)), f"call {call}, job {k}: absmax"
            assert np.float32(mu[0]).view(np.uint32) == np.float32(mu_ref).view(np.uint32), f"call {call}, job {k}: mu"
            assert np.array_equal(b.view(np.uint32), np.asarray(b_ref, np.float32).view(np.uint32)), \
                f"call {call}, job {k}: scales"
            assert np.array_equal(q, np.asarray(q_ref, np.int8)), f"call {call}, job {k}: qabs"
            assert _scratch_at_rest(ws[256 * k:256 * (k + 1)])
