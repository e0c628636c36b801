"""CPU oracle of the SS2D block around the core.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
CPU-baseline leg of bench.py, never by the product path.  Plain numpy in fp64;
the core itself is the C oracle's forward_core (oracle.py).  No blocking, no
fusion: each step below is one numpy expression over whole arrays.

What the block computes.  The SS2D article (section 1, "architecture
overview") lists the block's parts in order: an input projection that maps the
d_model features to the wider d_inner = D channels, a depthwise convolution
that captures local spatial features, the cross scan with the selective scan
(the core), and an output projection back to d_model.  The VMamba overview
page (section 2.2, the SS2D constructor) gives the activation (SiLU) and the
convolution's kernel size (d_conv = 3), and says that a learnable gate adjusts
the flow of information.  The pages print no forward pass for the block, so
the steps are read as follows (each reading is the plainest one the rest of
the pages support):

  1. xz = x @ W_in^T (+ b_in): x is (B, H, W, d_model), channels last (the
     article's default input layout, section 3.1); xz has 2D channels, the
     first D are the scan branch x_in and the last D the gate branch z.
  2. x_c = SiLU(depthwise_conv(x_in) + b_conv): a d_conv x d_conv kernel per
     channel, cross-correlation with zero padding (d_conv - 1) / 2, so the
     output keeps H x W.
  3. y = forward_core(x_c): the core, in its projection form (x_proj and
     dt_proj of section 3.2), channel-first.
  4. g = LayerNorm_D(y) * SiLU(z): the output normalisation over the D
     channels of each pixel (biased variance, eps inside the square root,
     affine weight and bias), gated by the z branch.
  5. out = g @ W_out^T (+ b_out): (B, H, W, d_model).

Precision (the article's mixed-precision advice, read as: bf16 storage between
the steps, wider arithmetic inside them): x, W_in, W_x and W_out are bf16
values; xz, x_c and g are rounded to bf16 (round to nearest, ties to even)
where they are stored; the core's output y and the block's output are kept
wide.  The oracle rounds at exactly those points and computes everything else
in fp64.
"""
from __future__ import annotations

import numpy as np

from . import oracle as _core


def round_bf16(a):
    """Nearest bfloat16 value of each element (ties to even), returned as fp64.

    A bf16 number is the top 16 bits of an IEEE binary32 number.  The value is
    first taken to binary32 (round to nearest), then the low 16 bits are
    rounded off: add 0x7FFF plus the lowest kept bit, and clear the low half."""
    a32 = np.ascontiguousarray(a, dtype=np.float32)
    bits = a32.view(np.uint32).astype(np.uint64)
    keep_lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + keep_lsb) & 0xFFFF0000).astype(np.uint32)
    return rounded.view(np.float32).astype(np.float64)


def silu(z):
    """SiLU(z) = z * sigmoid(z) = z / (1 + exp(-z)), the act_layer of the SS2D constructor."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def linear(a, weight, bias=None):
    """a (..., K) times weight (M, K) transposed, plus bias (M): a library matmul in fp64."""
    out = np.asarray(a, dtype=np.float64) @ np.asarray(weight, dtype=np.float64).T
    if bias is not None:
        out = out + np.asarray(bias, dtype=np.float64)
    return out


def depthwise_conv(x, weight, bias=None):
    """Depthwise 2-D cross-correlation of channels-last x (B, H, W, D) with one k x k kernel
    per channel (weight (D, k, k), k odd), zero padding (k - 1) / 2 on every side, so the
    output is (B, H, W, D):
        out[b, h, w, d] = sum_{i, j} weight[d, i, j] * x[b, h + i - r, w + j - r, d] + bias[d]
    with r = (k - 1) / 2 and x taken as zero outside the image."""
    x = np.asarray(x, dtype=np.float64)
    weight = np.asarray(weight, dtype=np.float64)
    B, H, W, D = x.shape
    k = weight.shape[1]
    assert weight.shape == (D, k, k) and k % 2 == 1
    r = (k - 1) // 2
    xp = np.zeros((B, H + 2 * r, W + 2 * r, D))
    xp[:, r:r + H, r:r + W, :] = x
    out = np.zeros((B, H, W, D))
    for i in range(k):
        for j in range(k):
            out += weight[:, i, j] * xp[:, i:i + H, j:j + W, :]
    if bias is not None:
        out += np.asarray(bias, dtype=np.float64)
    return out


def layer_norm(y, weight, bias, eps):
    """LayerNorm over the last axis: (y - mean) / sqrt(var + eps) * weight + bias, with the
    mean and the biased (population) variance of each row."""
    y = np.asarray(y, dtype=np.float64)
    mean = y.mean(axis=-1, keepdims=True)
    var = ((y - mean) ** 2).mean(axis=-1, keepdims=True)
    return (y - mean) / np.sqrt(var + eps) * np.asarray(weight, dtype=np.float64) + np.asarray(bias, dtype=np.float64)


def block_forward(x, in_proj_weight, conv_weight, conv_bias, x_proj_weight, dt_projs_weight, dt_projs_bias,
                  A_logs, Ds, out_norm_weight, out_norm_bias, out_proj_weight, in_proj_bias=None,
                  out_proj_bias=None, eps=1e-5, delta_softplus=True, intermediates=False, store_bf16=True):
    """The SS2D block of the module docstring.  x (B, H, W, d_model) -> out (B, H, W, d_model).

    Shapes: in_proj_weight (2D, d_model), conv_weight (D, k, k), conv_bias (D) or None,
    x_proj_weight (4, R + 2N, D), dt_projs_weight (4, D, R), dt_projs_bias (4D),
    A_logs (4D, N), Ds (4D), out_norm_weight / out_norm_bias (D), out_proj_weight (d_model, D).
    With intermediates=True also returns a dict of xz, x_c, y (channels last) and g.
    With store_bf16=False the three stored intermediates keep their fp64 values (no bf16
    rounding; x_c still enters the core as given), which measures how much the block's
    output depends on the rounding at its storage points."""
    rnd = round_bf16 if store_bf16 else (lambda v: v)
    x = np.asarray(x, dtype=np.float64)
    B, H, W, d_model = x.shape
    D = np.asarray(conv_weight).shape[0]
    assert np.asarray(in_proj_weight).shape == (2 * D, d_model)
    assert np.asarray(out_proj_weight).shape == (d_model, D)
    # 1. input projection, stored in bf16; the first D channels feed the scan, the last D the gate
    xz = rnd(linear(x, in_proj_weight, in_proj_bias))
    x_in, z = xz[..., :D], xz[..., D:]
    # 2. depthwise convolution and SiLU, stored in bf16
    x_c = rnd(silu(depthwise_conv(x_in, conv_weight, conv_bias)))
    # 3. the core (channel-first in the C oracle)
    y_cf = _core.forward_core(np.ascontiguousarray(x_c.transpose(0, 3, 1, 2)), A_logs, Ds, dt_projs_bias,
                              x_proj_weight=x_proj_weight, dt_projs_weight=dt_projs_weight,
                              delta_softplus=delta_softplus)
    y = y_cf.transpose(0, 2, 3, 1)
    # 4. output normalisation over D, gated by SiLU(z), stored in bf16
    g = rnd(layer_norm(y, out_norm_weight, out_norm_bias, eps) * silu(z))
    # 5. output projection
    out = linear(g, out_proj_weight, out_proj_bias)
    if intermediates:
        return out, dict(xz=xz, x_c=x_c, y=y, g=g)
    return out
