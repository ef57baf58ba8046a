"""Test-side glue: runs the CPU oracle on a synthetic workload and moves the
same seeded inputs to the GPU.  Expected values come only from ``oracle``."""
import numpy as np
import torch

from bit_nf4_quantized_07_b200 import synthetic
from oracle import codec, linear


def bf16_to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev_bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f64(bits):
    return codec.bf16_bits_to_f64(bits)


class OracleWeight:
    """NF4 + DQ of a fp32 weight by the oracle, with W' as BF16 bits."""

    def __init__(self, w: np.ndarray, double_quant: bool = True, dq_format: str = "int8"):
        self.rows, self.cols = w.shape
        self.numel = w.size
        self.codes, self.absmax = codec.quantize(w)
        self.dq = double_quant
        if double_quant:
            self.qabs, self.scale, self.mu = codec.double_quant(self.absmax, fmt=dq_format)
            self.wp_bits = codec.dequant(self.codes, self.numel, qabs=self.qabs, scale=self.scale, mu=self.mu,
                                         fmt=dq_format)
        else:
            self.wp_bits = codec.dequant(self.codes, self.numel, absmax=self.absmax)
        self.wp_bits = self.wp_bits.reshape(self.rows, self.cols)

    def wp_rows(self, r0, r1):
        return f64(self.wp_bits[r0:r1])


def forward_ref(ow: OracleWeight, X, A, B, s, token_idx=None, chunk=4096):
    """fp64 Y (rows ``token_idx`` or all) and U."""
    Xf, Af, Bf = f64(X), f64(A), f64(B)
    if token_idx is not None:
        Xf = Xf[token_idx]
    U = linear.lora_down(Xf, Af)
    Y = np.empty((Xf.shape[0], ow.rows))
    for r0 in range(0, ow.rows, chunk):
        r1 = min(ow.rows, r0 + chunk)
        Wp = ow.wp_rows(r0, r1)
        Y[:, r0:r1] = linear.forward(Wp, Xf, Af, Bf[r0:r1], s)[0]
    return Y, U


def backward_ref(ow: OracleWeight, X, A, B, s, dY, token_idx=None, chunk=4096):
    """fp64 dX (rows ``token_idx`` or all), dA, dB."""
    Xf, Af, Bf, dYf = f64(X), f64(A), f64(B), f64(dY)
    G = dYf @ Bf
    dA = s * (G.T @ Xf)
    dB = s * (dYf.T @ linear.lora_down(Xf, Af))
    rows = slice(None) if token_idx is None else token_idx
    dYs = dYf[rows]
    dX = s * (G[rows] @ Af)
    for r0 in range(0, ow.rows, chunk):
        r1 = min(ow.rows, r0 + chunk)
        dX += dYs[:, r0:r1] @ ow.wp_rows(r0, r1)
    # the full-tensor formula, for the dense (small) case
    if token_idx is None and ow.numel <= 1 << 22:
        dX_full, dA_full, dB_full = linear.backward(ow.wp_rows(0, ow.rows), Xf, Af, Bf, s, dYf)
        assert np.allclose(dX, dX_full) and np.allclose(dA, dA_full) and np.allclose(dB, dB_full)
    return dX, dA, dB


def workload(cfg: synthetic.LinearConfig):
    w = synthetic.weight_f32(cfg)
    X, A, B, dY = synthetic.activations_bf16(cfg)
    return w, X, A, B, dY
