"""The Sparse Transformer block around the attention op, in float64 (oracle).

Test infrastructure only (see the package docstring).

The pages describe the block only in words: a residual block with
pre-activation and layer normalisation, built so that very deep networks
train ("[논문 리뷰] Generating Long Sequences with Sparse Transformers",
"제안 방법", third item; the pcnews translation, "Глубокое внимание": the
order of operations inside the transformer was changed for depth), whose
attention and feed-forward parts are recomputed in the backward pass from
checkpoints instead of stored ("제안 방법", fourth item; ABSTRACT, item b;
"Глубокое внимание").  The readings taken where they are silent:

* pre-activation residual: each sub-block reads a layer-normalised copy of
  the residual stream and adds its output back to the stream unnormalised:
  ``h = x + attn(LN1(x))``, ``y = h + ff(LN2(h))``;
* layer normalisation over the model width C = H * D with a gain and a bias
  per channel, biased variance, epsilon 1e-5;
* ``attn(a) = concat_h(A_h) Wo`` with ``[q | k | v] = a Wqkv``, head h
  taking columns ``h*D .. h*D + D - 1`` of each of q, k, v, and ``A_h`` the
  causal factorized attention of ``oracle.attention`` (scale 1/sqrt(D));
* ``ff(f) = gelu(f W1) W2`` with a hidden width of 4C and the exact GELU
  ``u * Phi(u)`` (Phi the standard normal CDF);
* the projections carry no bias.

``backward`` returns the gradient of ``sum(y * dy)`` with respect to the
block input and every parameter, from the block input alone: it runs the
forward again (the recomputation), then the chain rule backwards, with the
layer-norm and GELU derivatives written out.
"""

import math

import numpy as np

from . import attention

EPS = 1e-5


def _erf(x):
    return np.vectorize(math.erf, otypes=[np.float64])(x)


def layer_norm(x, g, b):
    """Normalise the last axis: ``(x - mean) / sqrt(var + EPS) * g + b``."""
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    xh = (x - mu) / np.sqrt(var + EPS)
    return xh * g + b


def layer_norm_backward(x, g, dy):
    """(dx, dg, db) of ``layer_norm`` for the upstream gradient ``dy``."""
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + EPS)
    xh = (x - mu) * rstd
    dxh = dy * g
    dx = rstd * (dxh - dxh.mean(axis=-1, keepdims=True) - xh * (dxh * xh).mean(axis=-1, keepdims=True))
    red = tuple(range(x.ndim - 1))
    return dx, (dy * xh).sum(axis=red), dy.sum(axis=red)


def gelu(u):
    return 0.5 * u * (1.0 + _erf(u / math.sqrt(2.0)))


def gelu_grad(u):
    """d gelu / du = Phi(u) + u phi(u)."""
    return 0.5 * (1.0 + _erf(u / math.sqrt(2.0))) + u * np.exp(-0.5 * u * u) / math.sqrt(2.0 * math.pi)


def _heads(t, H):
    """``[B, N, C]`` -> ``[B, H, N, D]`` (head h = columns h*D .. h*D+D-1)."""
    B, N, C = t.shape
    return t.reshape(B, N, H, C // H).transpose(0, 2, 1, 3)


def _merge(t):
    """``[B, H, N, D]`` -> ``[B, N, H*D]``."""
    B, H, N, D = t.shape
    return t.transpose(0, 2, 1, 3).reshape(B, N, H * D)


def forward(x, p, H, mode, l=1, c=0):
    """Block output ``y`` and the intermediates (a dict) for input ``x``
    ``[B, N, C]`` and parameters ``p`` (keys ln1_g, ln1_b, w_qkv [C, 3C],
    w_o [C, C], ln2_g, ln2_b, w_1 [C, 4C], w_2 [4C, C])."""
    x = np.asarray(x, dtype=np.float64)
    p = {k: np.asarray(v, dtype=np.float64) for k, v in p.items()}
    C = x.shape[-1]
    a = layer_norm(x, p["ln1_g"], p["ln1_b"])
    qkv = a @ p["w_qkv"]
    q, k, v = (_heads(qkv[..., i * C:(i + 1) * C], H) for i in range(3))
    o, lse = attention.forward(q, k, v, mode, l, c)
    o2 = _merge(o)
    h = x + o2 @ p["w_o"]
    f = layer_norm(h, p["ln2_g"], p["ln2_b"])
    u = f @ p["w_1"]
    gl = gelu(u)
    y = h + gl @ p["w_2"]
    return y, dict(a=a, q=q, k=k, v=v, o=o, lse=lse, o2=o2, h=h, f=f, u=u, g=gl)


def backward(x, dy, p, H, mode, l=1, c=0):
    """``(dx, grads)`` for the upstream gradient ``dy`` of ``y``; grads has
    the keys of ``p``.  Only ``x`` is kept from the forward pass: every
    intermediate is computed again here."""
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    p = {k: np.asarray(v, dtype=np.float64) for k, v in p.items()}
    _, t = forward(x, p, H, mode, l, c)
    red = tuple(range(x.ndim - 1))

    def wgrad(inp, d):  # sum over rows of inp^T d
        return np.tensordot(inp, d, axes=(red, red))

    g = {}
    g["w_2"] = wgrad(t["g"], dy)
    dgl = dy @ p["w_2"].T
    du = dgl * gelu_grad(t["u"])
    g["w_1"] = wgrad(t["f"], du)
    df = du @ p["w_1"].T
    dh_ln, g["ln2_g"], g["ln2_b"] = layer_norm_backward(t["h"], p["ln2_g"], df)
    dh = dy + dh_ln
    g["w_o"] = wgrad(t["o2"], dh)
    do = _heads(dh @ p["w_o"].T, H)
    dq, dk, dv = attention.backward(t["q"], t["k"], t["v"], do, mode, l, c, lse=t["lse"])
    dqkv = np.concatenate([_merge(dq), _merge(dk), _merge(dv)], axis=-1)
    g["w_qkv"] = wgrad(t["a"], dqkv)
    da = dqkv @ p["w_qkv"].T
    dx_ln, g["ln1_g"], g["ln1_b"] = layer_norm_backward(x, p["ln1_g"], da)
    return dh + dx_ln, g
