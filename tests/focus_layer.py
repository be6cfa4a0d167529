"""A synthetic layer-output objective for the FOCUS calibration tests (test
helper, not a test module): the layer's weights, the Gram matrix of its
correlated synthetic inputs, and the loss with its gradient formed in float64
from the oracle's forward pass."""
import numpy as np

from microscaling_fp4_quantization_bf16_b200 import synth


def f32_of_bf16(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32)


def layer_problem(rows, cols, tokens, seed):
    """Synthetic layer: W ~ N(0, 0.02^2); inputs X with per-channel scales, a
    few outlier channels (x20) and mixed (correlated) channels; H = X^T X / T."""
    w = synth.gaussian(rows, cols, seed=seed, std=0.02)
    rng = np.random.default_rng(seed + 1)
    x = rng.standard_normal((tokens, cols)) * rng.uniform(0.1, 2.1, cols)
    x[:, rng.choice(cols, max(1, cols // 100), replace=False)] *= 20
    x = x @ (np.eye(cols) + 0.3 * rng.standard_normal((cols, cols)) / np.sqrt(cols))
    return synth.bits16(w), x.T @ x / tokens


def layer_loss_and_grad(ref, wb, c, h, fmt="nvfp4", block=16, sub=8):
    """L = tr(E H E^T) = |X E^T|^2 / T with E = W_hat - W (fp32 W_hat of the
    oracle's forward at fp16(c)); dL/dW_hat = 2 E H, rounded to bf16."""
    ch = np.asarray(c, np.float32).astype(np.float16).view(np.uint16)
    wh = ref.focus_fwd(wb, ch, fmt, block, sub, out="f32", want_codes=False)["w_hat"]
    e = wh.astype(np.float64) - f32_of_bf16(wb).astype(np.float64)
    eh = e @ h
    return float(np.sum(eh * e)), synth.bits16(synth.to_bf16(2 * eh))
