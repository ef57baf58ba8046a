"""Float64 oracle of the AdamW update of the LoRA factors (the optimizer the
QLoRA recipe pages with NVIDIA unified memory).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Pages followed:
  "QLoRA: Efficient Finetuning of Quantized LLMs" deck "3 QLoRA Finetuning",
      card 5: paged optimizers keep the optimizer states in NVIDIA unified
      memory, paged out to CPU RAM when the GPU runs short and paged back for
      the update; card 1: only the adapter parameters receive updates.
  "LoRA 与 QLoRA" (whoami-wesleyyou.top), QLoRA usage notes: the optimizer is
      paged_adamw_32bit (32-bit AdamW states), gradients and AdamW states only
      for the LoRA parameters.
The pages do not write AdamW out.  This follows the published algorithm,
Loshchilov & Hutter, "Decoupled Weight Decay Regularization" (ICLR 2019),
Algorithm 2 with a constant schedule multiplier, in the form PyTorch's
torch.optim.AdamW uses (weight decay applied to the parameter before the
adaptive step; bias corrections on m and v):

  t >= 1 (the step being taken)
  m_t = b1 m_{t-1} + (1 - b1) g
  v_t = b2 v_{t-1} + (1 - b2) g^2
  p  <- p (1 - lr wd)
  p  <- p - lr * (m_t / (1 - b1^t)) / (sqrt(v_t / (1 - b2^t)) + eps)

Parity status: pinned against torch.optim.AdamW (float64) and the closed
forms of the first step and of a constant gradient; the reading that the
LoRA factors keep fp32 master copies (written back to BF16 for the forward)
is ours.
"""
import numpy as np


def adamw_step(p, g, m, v, t, lr, b1=0.9, b2=0.999, eps=1e-8, wd=0.0):
    """One AdamW step in float64.  Returns (p, m, v), new arrays."""
    p = np.asarray(p, np.float64)
    g = np.asarray(g, np.float64)
    m = b1 * np.asarray(m, np.float64) + (1.0 - b1) * g
    v = b2 * np.asarray(v, np.float64) + (1.0 - b2) * g * g
    p = p * (1.0 - lr * wd)
    mhat = m / (1.0 - b1 ** t)
    vhat = v / (1.0 - b2 ** t)
    p = p - lr * mhat / (np.sqrt(vhat) + eps)
    return p, m, v
