"""GPU parity of the fused QLoRA linear (forward and backward) against the
float64 oracle.  Tolerance (the stated target): normwise max relative error
max|T - T*| / max|T*| <= 2e-2 per output tensor."""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_07_b200 import api, synthetic
from oracle import linear
from tests.oracle_ref import (OracleWeight, backward_ref, bf16_to_dev, dev_bf16_bits, f64, forward_ref,
                              workload)

pytestmark = pytest.mark.gpu
TOL = 2e-2


def _gpu_weight(w, double_quant=True, dq_format="int8"):
    return api.quantize_weight(torch.from_numpy(w).cuda(), double_quant=double_quant, dq_format=dq_format)


def _run(cfg, w, X, A, B, dY, double_quant=True, backward=True, dq_format="int8"):
    wq = _gpu_weight(w, double_quant, dq_format)
    Xd, Ad, Bd = bf16_to_dev(X), bf16_to_dev(A), bf16_to_dev(B)
    Y, U = api.qlora_linear_fwd(wq, Xd, Ad, Bd, cfg.s)
    out = {"Y": f64(dev_bf16_bits(Y)), "U": f64(dev_bf16_bits(U))}
    if backward:
        dX, dA, dB = api.qlora_linear_bwd(wq, Xd, Ad, Bd, cfg.s, bf16_to_dev(dY), U=U)
        out.update(dX=f64(dev_bf16_bits(dX)), dA=dA.double().cpu().numpy(), dB=dB.double().cpu().numpy())
    torch.cuda.synchronize()
    return out


def _compare(name, got, ref, tol=TOL):
    err = linear.normwise_error(got, ref)
    fro = linear.frobenius_error(got, ref)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), name
    assert err <= tol, f"{name}: normwise {err:.3e} (frobenius {fro:.3e})"
    return err


SMALL = [
    synthetic.PR1,
    synthetic.custom("ragged_192x320_n77_r16", 192, 320, 77, 16, s=2.0, index=11),
    synthetic.custom("single_token_128x128_n1_r8", 128, 128, 1, 8, s=0.5, index=12),
    synthetic.custom("tall_256x512_n300_r64", 256, 512, 300, 64, s=1.0, index=13),
    synthetic.custom("r128_128x256_n33_r128", 128, 256, 33, 128, s=2.0, index=14),
    synthetic.custom("tokens_tile_512x256_n256_r16", 512, 256, 256, 16, s=2.0, index=15),
    synthetic.custom("wide_384x1024_n640_r32", 384, 1024, 640, 32, s=1.5, index=16, outlier_rate=0.001),
    # tcgen05 path with r = 128: dA and dB beside the dX GEMM with 16 fragment columns
    synthetic.custom("side_r128_256x512_n128_r128", 256, 512, 128, 128, s=0.5, index=42),
    # ragged token tiles on the tcgen05 path, side kernel with r = 24
    synthetic.custom("side_r24_640x768_n200_r24", 640, 768, 200, 24, s=1.0, index=43),
]


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
@pytest.mark.parametrize("dq", [True, False], ids=["dq", "plain"])
def test_linear_small_configs(cfg, dq):
    w, X, A, B, dY = workload(cfg)
    ow = OracleWeight(w, double_quant=dq)
    got = _run(cfg, w, X, A, B, dY, double_quant=dq)
    Y, U = forward_ref(ow, X, A, B, cfg.s)
    dX, dA, dB = backward_ref(ow, X, A, B, cfg.s, dY)
    _compare("U", got["U"], U)
    _compare("Y", got["Y"], Y)
    _compare("dX", got["dX"], dX)
    _compare("dA", got["dA"], dA)
    _compare("dB", got["dB"], dB)


@pytest.mark.parametrize("batch", [1, 4, 16])
def test_decode_forward(batch):
    cfg = synthetic.DECODE[batch]
    w, X, A, B, dY = workload(cfg)
    ow = OracleWeight(w)
    got = _run(cfg, w, X, A, B, dY, backward=False)
    Y, U = forward_ref(ow, X, A, B, cfg.s)
    _compare("U", got["U"], U)
    _compare("Y", got["Y"], Y)


DECODE_SHAPES = [
    synthetic.custom("dec_8192x512_n24_r32", 8192, 512, 24, 32, s=1.5, index=21),    # >1 row group per CTA
    synthetic.custom("dec_4096x1024_n32_r128", 4096, 1024, 32, 128, s=0.5, index=22),
    synthetic.custom("dec_1024x4096_n5_r8", 1024, 4096, 5, 8, s=2.0, index=23),
    synthetic.custom("dec_256x2048_n9_r16", 256, 2048, 9, 16, s=2.0, index=24),
    synthetic.custom("dec_128x11008_n3_r24", 128, 11008, 3, 24, s=1.0, index=25),   # ragged K ranges, 3 U warp columns
    synthetic.custom("dec_64x64_n32_r8", 64, 64, 32, 8, s=2.0, index=26),           # one block: empty U sub-ranges
    synthetic.custom("dec_512x768_n17_r40", 512, 768, 17, 40, s=0.5, index=27),     # 3 token tiles, r % 16 == 8
    synthetic.custom("dec_1024x1536_n25_r64", 1024, 1536, 25, 64, s=1.5, index=28), # 4 token tiles
]


@pytest.mark.parametrize("cfg", DECODE_SHAPES, ids=lambda c: c.name)
@pytest.mark.parametrize("dq", [True, False], ids=["dq", "plain"])
def test_decode_shaped_forward(cfg, dq):
    w, X, A, B, dY = workload(cfg)
    ow = OracleWeight(w, double_quant=dq)
    got = _run(cfg, w, X, A, B, dY, double_quant=dq, backward=False)
    Y, U = forward_ref(ow, X, A, B, cfg.s)
    _compare("U", got["U"], U)
    _compare("Y", got["Y"], Y)


def test_decode_forward_right_behind_the_quantize_sees_its_outputs():
    """The decode forward enqueued directly behind nf4_quantize_dq on the same
    stream, with no synchronisation between, reads the fresh codes, scales
    and mean: every read of the weight comes after its dependency wait.  The
    output buffers hold wrong values (a mean of 123) before each quantize; the
    result must equal that of a forward run after the stream has drained, and
    the oracle's."""
    cfg = synthetic.DECODE[4]
    w, X, A, B, dY = workload(cfg)
    Wd = torch.from_numpy(w).cuda()
    wq = api.quantize_weight(Wd)
    Xd, Ad, Bd = bf16_to_dev(X), bf16_to_dev(A), bf16_to_dev(B)
    ws = api.alloc_workspace(api.workspace_bytes(api.OP_LINEAR_FWD, cfg.dout, cfg.din, cfg.n, cfg.r))
    torch.cuda.synchronize()
    Yref, Uref = api.qlora_linear_fwd(wq, Xd, Ad, Bd, cfg.s, ws=ws)
    torch.cuda.synchronize()
    for _ in range(4):
        wq.dq_mean.fill_(123.0)
        wq.dq_scale.fill_(7.0)
        wq.qabs.fill_(-100)
        api.nf4_quantize_dq(Wd, wq.codes, wq.absmax, wq.qabs, wq.dq_scale, wq.dq_mean)
        Y, U = api.qlora_linear_fwd(wq, Xd, Ad, Bd, cfg.s, ws=ws)
        torch.cuda.synchronize()
        assert torch.equal(Y, Yref) and torch.equal(U, Uref)
    assert api.device_status(ws) == 0
    Yo, _ = forward_ref(OracleWeight(w), X, A, B, cfg.s)
    _compare("Y", f64(dev_bf16_bits(Y)), Yo)


def test_decode_forward_repeats_and_replays_bit_identically():
    """The one-launch decode forward folds its split-K partials in an order
    fixed by the shape: back-to-back calls on one workspace, a call after a
    backward on the same workspace, and CUDA graph replays must all give the
    same bits."""
    cfg = synthetic.custom("rep_1024x2048_n12_r16", 1024, 2048, 12, 16, s=2.0, index=29)
    w, X, A, B, dY = workload(cfg)
    wq = _gpu_weight(w)
    Xd, Ad, Bd, dYd = bf16_to_dev(X), bf16_to_dev(A), bf16_to_dev(B), bf16_to_dev(dY)
    nbytes = max(api.workspace_bytes(api.OP_LINEAR_FWD, cfg.dout, cfg.din, cfg.n, cfg.r),
                 api.workspace_bytes(api.OP_LINEAR_BWD, cfg.dout, cfg.din, cfg.n, cfg.r))
    ws = api.alloc_workspace(nbytes)
    Y0, U0 = api.qlora_linear_fwd(wq, Xd, Ad, Bd, cfg.s, ws=ws)
    for _ in range(3):
        Y1, U1 = api.qlora_linear_fwd(wq, Xd, Ad, Bd, cfg.s, ws=ws)
        assert torch.equal(Y0, Y1) and torch.equal(U0, U1)
    api.qlora_linear_bwd(wq, Xd, Ad, Bd, cfg.s, dYd, U=U0, ws=ws)
    Y2, U2 = api.qlora_linear_fwd(wq, Xd, Ad, Bd, cfg.s, ws=ws)
    assert torch.equal(Y0, Y2) and torch.equal(U0, U2)
    assert api.device_status(ws) == 0
    Yg = torch.empty_like(Y0)
    Ug = torch.empty_like(U0)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        api.qlora_linear_fwd(wq, Xd, Ad, Bd, cfg.s, Y=Yg, U_out=Ug, ws=ws)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(4):
            api.qlora_linear_fwd(wq, Xd, Ad, Bd, cfg.s, Y=Yg, U_out=Ug, ws=ws)
    Yg.zero_()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(Y0, Yg) and torch.equal(U0, Ug)
    got = {"Y": f64(dev_bf16_bits(Yg)), "U": f64(dev_bf16_bits(Ug))}
    Y, U = forward_ref(OracleWeight(w), X, A, B, cfg.s)
    _compare("U", got["U"], U)
    _compare("Y", got["Y"], Y)


def test_adapter_off_matches_cublas_on_materialised_weight():
    """B = 0 (or s = 0): the fused forward reduces to X W'^T; cross-check it
    against torch.matmul (cuBLAS) on nf4_dequant's materialised W'."""
    cfg = synthetic.custom("b0_512x512_n96", 512, 512, 96, 16, index=17)
    w, X, A, B, dY = workload(cfg)
    wq = _gpu_weight(w)
    Xd, Ad = bf16_to_dev(X), bf16_to_dev(A)
    Y0, _ = api.qlora_linear_fwd(wq, Xd, Ad, torch.zeros(cfg.dout, cfg.r, dtype=torch.bfloat16, device="cuda"), 2.0)
    Ys, _ = api.qlora_linear_fwd(wq, Xd, Ad, bf16_to_dev(B), 0.0)
    ref = torch.matmul(Xd.float(), api.nf4_dequant(wq).float().T)
    for Y in (Y0, Ys):
        err = (Y.float() - ref).abs().max().item() / ref.abs().max().item()
        assert err <= 4e-3, err


def test_backward_with_and_without_saved_u_and_determinism():
    cfg = synthetic.custom("reuse_256x256_n100_r16", 256, 256, 100, 16, index=18)
    w, X, A, B, dY = workload(cfg)
    wq = _gpu_weight(w)
    Xd, Ad, Bd, dYd = bf16_to_dev(X), bf16_to_dev(A), bf16_to_dev(B), bf16_to_dev(dY)
    Y1, U = api.qlora_linear_fwd(wq, Xd, Ad, Bd, cfg.s)
    Y2, _ = api.qlora_linear_fwd(wq, Xd, Ad, Bd, cfg.s)
    assert torch.equal(Y1, Y2)
    a = api.qlora_linear_bwd(wq, Xd, Ad, Bd, cfg.s, dYd, U=U)
    b = api.qlora_linear_bwd(wq, Xd, Ad, Bd, cfg.s, dYd, U=None)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_all_zero_weight_leaves_only_the_adapter():
    cfg = synthetic.custom("zero_w_128x192_n40_r8", 128, 192, 40, 8, index=19)
    _, X, A, B, dY = workload(cfg)
    w = np.zeros((cfg.dout, cfg.din), np.float32)
    got = _run(cfg, w, X, A, B, dY)
    U = f64(X) @ f64(A).T
    _compare("Y", got["Y"], cfg.s * U @ f64(B).T)


def _sampled(cfg, ntok=8):
    w, X, A, B, dY = workload(cfg)
    ow = OracleWeight(w)
    got = _run(cfg, w, X, A, B, dY)
    rng = np.random.Generator(np.random.PCG64(cfg.index))
    tok = np.unique(np.r_[0, cfg.n - 1, rng.integers(0, cfg.n, ntok)])
    Y, U = forward_ref(ow, X, A, B, cfg.s, token_idx=tok)
    _compare("U", got["U"][tok], U)
    _compare("Y", got["Y"][tok], Y)
    dX, dA, dB = backward_ref(ow, X, A, B, cfg.s, dY, token_idx=tok)
    _compare("dX", got["dX"][tok], dX)
    _compare("dA", got["dA"], dA)
    _compare("dB", got["dB"], dB)


def test_prefill_sampled():
    _sampled(synthetic.PREFILL)


@pytest.mark.slow
def test_large_sampled():
    _sampled(synthetic.LARGE)


E4M3_SHAPES = [
    synthetic.custom("e4m3_tc_512x768_n256_r16", 512, 768, 256, 16, s=2.0, index=31),    # tcgen05 path
    synthetic.custom("e4m3_mma_256x320_n40_r8", 256, 320, 40, 8, s=1.0, index=32),       # mma.sync path
    synthetic.custom("e4m3_dec_1024x2048_n4_r16", 1024, 2048, 4, 16, s=2.0, index=33),  # decode kernel
]


@pytest.mark.parametrize("cfg", E4M3_SHAPES, ids=lambda c: c.name)
def test_linear_with_e4m3_double_quant(cfg):
    """Every fused path restores the block constants from E4M3 codes when the
    weight says so: forward and backward within the tolerance of the oracle's
    E4M3-restored W'."""
    w, X, A, B, dY = workload(cfg)
    ow = OracleWeight(w, dq_format="e4m3")
    got = _run(cfg, w, X, A, B, dY, dq_format="e4m3")
    Y, U = forward_ref(ow, X, A, B, cfg.s)
    dX, dA, dB = backward_ref(ow, X, A, B, cfg.s, dY)
    _compare("U", got["U"], U)
    _compare("Y", got["Y"], Y)
    _compare("dX", got["dX"], dX)
    _compare("dA", got["dA"], dA)
    _compare("dB", got["dB"], dB)


def test_decode_forward_needs_no_zeroed_workspace():
    """The decode-sized forward keeps no state in the workspace: a header full
    of stale values (an old QLN_ERR_TIMEOUT in the status word, nonzero bytes
    everywhere) is cleared by the call's first CTA, and the result is exact."""
    cfg = synthetic.custom("stale_ws_1024x2048_n4_r16", 1024, 2048, 4, 16, s=2.0, index=41)
    w, X, A, B, dY = workload(cfg)
    wq = _gpu_weight(w)
    Xd, Ad, Bd = bf16_to_dev(X), bf16_to_dev(A), bf16_to_dev(B)
    ws = api.alloc_workspace(api.workspace_bytes(api.OP_LINEAR_FWD, cfg.dout, cfg.din, cfg.n, cfg.r))
    ws.fill_(0x5A)
    ws[0:4].view(torch.int32).fill_(7)
    Y, U = api.qlora_linear_fwd(wq, Xd, Ad, Bd, cfg.s, ws=ws)
    torch.cuda.synchronize()
    assert api.device_status(ws) == 0
    Yr, Ur = forward_ref(OracleWeight(w), X, A, B, cfg.s)
    _compare("U", f64(dev_bf16_bits(U)), Ur)
    _compare("Y", f64(dev_bf16_bits(Y)), Yr)


@pytest.mark.parametrize("batch", [1, 16])
def test_decode_forwards_on_two_unordered_streams(batch):
    """Two decode-sized forwards enqueued on two streams with no order between
    them, each a grid of one CTA per SM: no CTA of either waits on a CTA
    outside its own cluster, so they finish in any interleaving and both match
    the oracle (and the same call made alone, bit for bit)."""
    cfgs = [synthetic.custom(f"conc{batch}_{i}_2048x4096_r16", 2048, 4096, batch, 16, s=2.0, index=44 + i)
            for i in range(2)]
    runs = []
    for cfg in cfgs:
        w, X, A, B, dY = workload(cfg)
        runs.append((cfg, w, X, A, B, _gpu_weight(w), bf16_to_dev(X), bf16_to_dev(A), bf16_to_dev(B)))
    alone = [api.qlora_linear_fwd(wq, Xd, Ad, Bd, cfg.s) for (cfg, _, _, _, _, wq, Xd, Ad, Bd) in runs]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = []
    for _ in range(3):
        for st in streams:
            st.wait_stream(torch.cuda.current_stream())
        res = [None, None]
        wss = [api.alloc_workspace(api.workspace_bytes(api.OP_LINEAR_FWD, c.dout, c.din, c.n, c.r)) for c, *_ in runs]
        torch.cuda.synchronize()
        for i, (st, run) in enumerate(zip(streams, runs)):
            cfg, _, _, _, _, wq, Xd, Ad, Bd = run
            with torch.cuda.stream(st):
                res[i] = (api.qlora_linear_fwd(wq, Xd, Ad, Bd, cfg.s, ws=wss[i]), wss[i])
        torch.cuda.synchronize()
        outs.append(res)
    for res in outs:
        for i, ((Y, U), ws) in enumerate(res):
            assert api.device_status(ws) == 0
            assert torch.equal(Y, alone[i][0]) and torch.equal(U, alone[i][1])
    for i, (cfg, w, X, A, B, *_rest) in enumerate(runs):
        Yr, Ur = forward_ref(OracleWeight(w), X, A, B, cfg.s)
        _compare("U", f64(dev_bf16_bits(alone[i][1])), Ur)
        _compare("Y", f64(dev_bf16_bits(alone[i][0])), Yr)


def test_backwards_on_two_unordered_streams_and_in_a_graph():
    """dA and dB run beside the dX GEMM as its programmatic dependent on the
    caller's own stream (no internal stream): two backward calls enqueued on
    two streams with no order between them, and the same call captured in a
    CUDA graph on a third stream, all match the call made alone bit for bit
    and the oracle within the tolerance."""
    cfgs = [synthetic.custom(f"bwd_conc_{i}_1024x1024_n512_r16", 1024, 1024, 512, 16, s=2.0, index=46 + i)
            for i in range(2)]
    runs = []
    for cfg in cfgs:
        w, X, A, B, dY = workload(cfg)
        wq = _gpu_weight(w)
        args = (wq, bf16_to_dev(X), bf16_to_dev(A), bf16_to_dev(B), cfg.s, bf16_to_dev(dY))
        runs.append((cfg, w, X, A, B, dY, args))
    alone = [api.qlora_linear_bwd(*a) for (*_, a) in runs]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for st in streams:
        st.wait_stream(torch.cuda.current_stream())
    res = [None, None]
    for i, st in enumerate(streams):
        with torch.cuda.stream(st):
            res[i] = api.qlora_linear_bwd(*runs[i][-1])
    torch.cuda.synchronize()
    for i in range(2):
        for x, y in zip(res[i], alone[i]):
            assert torch.equal(x, y)
    # captured on a side stream, replayed twice
    wq, Xd, Ad, Bd, s_, dYd = runs[0][-1]
    cfg = runs[0][0]
    dX = torch.empty(cfg.n, cfg.din, dtype=torch.bfloat16, device="cuda")
    dA = torch.empty(cfg.r, cfg.din, dtype=torch.float32, device="cuda")
    dB = torch.empty(cfg.dout, cfg.r, dtype=torch.float32, device="cuda")
    ws = api.alloc_workspace(api.workspace_bytes(api.OP_LINEAR_BWD, cfg.dout, cfg.din, cfg.n, cfg.r))
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        api.qlora_linear_bwd(wq, Xd, Ad, Bd, s_, dYd, dX=dX, dA=dA, dB=dB, ws=ws)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        api.qlora_linear_bwd(wq, Xd, Ad, Bd, s_, dYd, dX=dX, dA=dA, dB=dB, ws=ws)
    for t in (dX, dA, dB):
        t.zero_()
    graph.replay()
    graph.replay()
    torch.cuda.synchronize()
    for x, y in zip((dX, dA, dB), alone[0]):
        assert torch.equal(x, y)
    for i, (cfg, w, X, A, B, dY, _) in enumerate(runs):
        dXr, dAr, dBr = backward_ref(OracleWeight(w), X, A, B, cfg.s, dY)
        _compare("dX", f64(dev_bf16_bits(alone[i][0])), dXr)
        _compare("dA", alone[i][1].double().cpu().numpy(), dAr)
        _compare("dB", alone[i][2].double().cpu().numpy(), dBr)


ADAPTER_CASES = [synthetic.DECODE[4],                                               # the decode-sized kernel
                 synthetic.custom("adapter_tc_1024x2048_n512_r16", 1024, 2048, 512, 16, s=2.0, index=48)]  # tcgen05


@pytest.mark.parametrize("cfg", ADAPTER_CASES, ids=lambda c: c.name)
def test_adapter_terms_alone(cfg):
    """The adapter term on its own ("LoRA 与 QLoRA", section LoRA: y = W0 x +
    s B(A x)): Y(B) - Y(B = 0) against the oracle's s U B^T, and dX(B) - dX(B = 0)
    against s G A with G = dY B, each normwise against its own magnitude.  B is
    drawn with sigma 0.5 (25 to 50 times the workload's) so the adapter term is
    about as large as the frozen-weight term.  Tolerance: the 2e-2 target plus the two bf16
    roundings of the outputs being subtracted (half an ulp each, at most 2^-9
    of the larger output), relative to the adapter term's magnitude."""
    w, X, A, _, dY = workload(cfg)
    B = synthetic.to_bf16_bits(synthetic.normal_f32((cfg.dout, cfg.r), 0.5, 4800 + cfg.index))
    wq = _gpu_weight(w)
    Xd, Ad, Bd, dYd = bf16_to_dev(X), bf16_to_dev(A), bf16_to_dev(B), bf16_to_dev(dY)
    B0 = torch.zeros_like(Bd)
    Y1, U1 = api.qlora_linear_fwd(wq, Xd, Ad, Bd, cfg.s)
    Y0, _ = api.qlora_linear_fwd(wq, Xd, Ad, B0, cfg.s)
    dX1, _, _ = api.qlora_linear_bwd(wq, Xd, Ad, Bd, cfg.s, dYd, U=U1)
    dX0, _, _ = api.qlora_linear_bwd(wq, Xd, Ad, B0, cfg.s, dYd, U=U1)
    torch.cuda.synchronize()
    Xf, Af, Bf, dYf = f64(X), f64(A), f64(B), f64(dY)
    for name, (t1, t0), ref in (("Y adapter", (Y1, Y0), cfg.s * (Xf @ Af.T) @ Bf.T),
                                ("dX adapter", (dX1, dX0), cfg.s * (dYf @ Bf) @ Af)):
        a1, a0 = f64(dev_bf16_bits(t1)), f64(dev_bf16_bits(t0))
        scale = np.max(np.abs(ref))
        tol = TOL + 2.0 ** -9 * (np.max(np.abs(a1)) + np.max(np.abs(a0))) / scale
        assert scale > 0.5 * np.max(np.abs(a0)), (name, "adapter term too small to test")
        _compare(name, a1 - a0, ref, tol=tol)
