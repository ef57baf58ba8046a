"""Float64 oracle of the QLoRA linear layer, forward and backward.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Layout (token-major, as the library stores it):
  X  [n][din]   activations       (the pages' x in R^{din x dseq}, transposed)
  W' [dout][din] doubleDequant(W0), the frozen weight as the matmul sees it
  A  [r][din],  B [dout][r]        the LoRA factors
  Y  [n][dout], U = X A^T [n][r]

Pages followed:
  "LoRA 与 QLoRA" (whoami-wesleyyou.top), section LoRA:
      Delta W = s B A;  y = W0 x + s B (A x);  W0 fixed, only A and B trained;
      rank(BA) <= r (section "rank 的证明").
  "QLoRA: Efficient Finetuning of Quantized LLMs" deck "3 QLoRA Finetuning",
      card 1: the matmul uses the dequantized BF16 weight; gradients flow
      through it, only the adapters receive updates.
  jjjymmm.cn 2024/03 QLoRA post, section "QLoRA": forward uses doubleDequant(W)
      with BF16 X; backward updates only the LoRA factors.

Every routine below is the textbook derivative of the scalar loss
L = sum(dY * Y) written out in float64 with NumPy matmuls; no intermediate
rounding (the GPU path rounds U, G and the outputs to its storage types).
"""
import numpy as np


def lora_down(X, A):
    """U = X A^T: the pages' A x for every token (n x r)."""
    return X @ A.T


def forward(Wp, X, A, B, s):
    """Y = X W'^T + s (X A^T) B^T  ("LoRA 与 QLoRA": y = W0 x + s B(A x)).

    Returns (Y, U)."""
    U = lora_down(X, A)
    return X @ Wp.T + s * (U @ B.T), U


def backward(Wp, X, A, B, s, dY):
    """Gradients of L = sum(dY * Y) for Y = forward(...).

    dX = dY W' + s (dY B) A      (flows through the dequantized weight)
    dA = s (dY B)^T X
    dB = s dY^T (X A^T)
    W0 gets no gradient (frozen).  Returns (dX, dA, dB)."""
    G = dY @ B
    dX = dY @ Wp + s * (G @ A)
    dA = s * (G.T @ X)
    dB = s * (dY.T @ lora_down(X, A))
    return dX, dA, dB


def merged_forward(Wp, X, A, B, s):
    """The same map through the merged weight W' + Delta W, Delta W = s B A
    ("LoRA 与 QLoRA", section LoRA).  Used only to cross-check ``forward``."""
    return X @ (Wp + s * (B @ A)).T


def normwise_error(T, Tref):
    """max|T - T*| / max|T*| (0 if both are zero)."""
    T = np.asarray(T, np.float64)
    Tref = np.asarray(Tref, np.float64)
    den = np.max(np.abs(Tref)) if Tref.size else 0.0
    num = np.max(np.abs(T - Tref)) if T.size else 0.0
    if den == 0.0:
        return float(num)
    return float(num / den)


def frobenius_error(T, Tref):
    T = np.asarray(T, np.float64)
    Tref = np.asarray(Tref, np.float64)
    den = np.linalg.norm(Tref)
    num = np.linalg.norm(T - Tref)
    return float(num / den) if den else float(num)
