"""Plain float64 CPU oracle of the ViT vision tower and its 2x2-merge projector.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this module.  The CUDA library never calls it, and it
shares no code with the CUDA library: it imports numpy and nothing else.

Every function is the plain definition of one step, in float64, in raster token order
(token (t, h, w) at index t*gh*gw + h*gw + w), written to be checked by eye against
the passage it cites.  Inputs are the same seeded numbers the GPU receives: bf16
weights and activations converted exactly to float64, fp32 pixels converted to float64.
The oracle rounds nothing itself.

Sources (web pages on the MiniMax-M3 vision tower):
  * "MiniMax-M3 Vision" model card, Architecture table: CLIP-style ViT, 32 layers,
    hidden 1280, 16 heads, intermediate 5120, patch 14, Conv3d patch embed, 3D RoPE,
    GELU; 2x2 spatial merge with temporal patch 2; projector Linear(1280,6144), GELU,
    Linear(6144,6144), flatten four 6144-wide patches, Linear(24576,6144), GELU,
    Linear(6144,6144).  Same card, Architecture notes: 1280-wide tower tokens,
    5120-wide merged tokens (2x2 of 1280), 6144-wide projected tokens at 448.
  * "v2_loaders - Differentiable Vision Tower Loaders (spark2)", section 3 (MiniMax-M3
    vision tower): the frame is repeated to temporal depth 2, grid_thw = [t, h, w],
    3D RoPE with rope_theta 10000.
  * "spark_model/layers/vision_encoder/enc_impl/init.rs" (VisionEncoder::new): per-axis
    RoPE inverse frequencies inv_freq[k] = theta^(-2k/dim), k < dim/2; ViT attention
    over a full [seq, seq] score matrix per head, i.e. the dense, non-causal softmax.
  * "metrale_model_arch/weight_loader/qwen3_vl.rs" (load_vision_encoder): a ViT block
    holds norm1, qkv, proj, norm2, fc1, fc2, each with weight and bias (pre-LN block).

Readings where the pages are silent (each is also checked by a pin in
tests/test_oracle_pins.py):
  * 3D RoPE: head channels split into contiguous blocks [t | h | w] of sizes
    ``rope_sections``; inside a block of size s, channel pair (j, j + s/2) is rotated
    by angle pos_axis * theta^(-2j/s) (rotate-half pairing).  Image positions are
    (t=0, h=row, w=col).
  * LayerNorm eps 1e-6, GELU in its tanh form, no CLS token, no absolute position
    embedding, no LayerNorm before or after the tower.
  * 2x2 merge: merged token (i, j) concatenates tokens (2i,2j), (2i,2j+1), (2i+1,2j),
    (2i+1,2j+1) in that order; merged tokens are in raster (i, j) order.
  * Images of a batch are independent (attention never crosses images).
  * Backward ("differentiable" loaders whose probe backpropagates the pooled tower
    feature, findings summary and section 3): the gradient of a scalar loss with respect
    to the model pixels, given its gradient with respect to the tower output, through
    every layer and the patch embedding (the chain rule applied to the forward above;
    weights are constants).
  * Preprocessing ("bicubic resize to 672x672, OpenAI CLIP mean/std", findings section
    3): the resize is separable cubic-convolution resampling with the Keys kernel at
    a = -0.5, output pixel centres mapped onto input pixel centres, the kernel widened
    by the scale factor when shrinking, taps outside the image dropped and the weights
    renormalised; resized values stay real numbers (no clamping or rounding to 8 bits)
    before scaling by 1/255 and normalising per channel.

Parity with the real MiniMax-M3 weights is not checked here (no trained weights or
reference outputs exist on the pages); every function below is pinned against
mathematics, library routines or brute force in the pin tests.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "token_grid", "patch_unfold", "patch_embed", "layer_norm", "gelu",
    "rope_inv_freq", "positions_raster", "apply_rope_3d", "attention",
    "attention_probs", "tower_layer", "tower_layer_rows", "merge_2x2", "projector",
    "patch_unfold_video", "forward_video",
    "cubic_kernel", "resize_taps", "resize_bicubic", "preprocess",
    "layer_norm_backward", "gelu_backward", "rope_3d_backward", "attention_backward",
    "tower_layer_backward", "patch_fold", "tower_backward",
    "projector_rows", "forward",
    "block_order", "merge_source_map",
]


# ----------------------------------------------------------------------- shapes

def token_grid(image_hw: tuple[int, int], patch: int = 14, merge: int = 2,
               frames: int = 1, temporal_patch: int = 2) -> dict:
    """Token counts of one image (model card, Architecture: patch 14, 2x2 merge).

    A single frame is repeated up to ``temporal_patch`` frames (v2_loaders FINDINGS,
    section 3), so one image gives t = 1.
    """
    H, W = image_hw
    if H % (patch * merge) or W % (patch * merge):
        raise ValueError("image side must be a multiple of patch * merge")
    t = max(1, -(-frames // temporal_patch))
    gh, gw = H // patch, W // patch
    n = t * gh * gw
    return dict(t=t, h=gh, w=gw, tokens=n, merged=n // (merge * merge))


# ----------------------------------------------------------- patch embedding

def patch_unfold(image: np.ndarray, patch: int = 14, temporal_patch: int = 2) -> np.ndarray:
    """One image [3, H, W] -> patch vectors [gh*gw, 3*tp*patch*patch] in raster order.

    v2_loaders FINDINGS, section 3: the temporal dimension is padded to 2 by repeating
    the frame.  Model card, Architecture: Conv3d patch embedding with patch 14 and
    temporal patch 2.  The vector of patch (h, w) lists the pixels in (c, t, kh, kw)
    order, the order of a Conv3d weight [hidden, 3, tp, patch, patch] flattened.
    """
    C, H, W = image.shape
    gh, gw = H // patch, W // patch
    out = np.empty((gh * gw, C * temporal_patch * patch * patch), dtype=np.float64)
    for h in range(gh):
        for w in range(gw):
            block = image[:, h * patch:(h + 1) * patch, w * patch:(w + 1) * patch]
            clip = np.stack([block] * temporal_patch, axis=1)  # [C, tp, p, p]
            out[h * gw + w] = clip.reshape(-1)
    return out


def patch_unfold_video(frames: np.ndarray, patch: int = 14, temporal_patch: int = 2) -> np.ndarray:
    """A clip [F, 3, H, W] -> patch vectors [T*gh*gw, 3*tp*patch*patch], raster (t, h, w).

    Temporal patch t covers frames t*tp .. t*tp + tp - 1 (model card, Architecture:
    temporal patch size 2); a clip whose frame count is not a multiple of tp repeats
    its last frame, the same rule that makes one image a clip of tp copies of its frame
    (v2_loaders FINDINGS, section 3).  T = ceil(F / tp).
    """
    F, C, H, W = frames.shape
    T = -(-F // temporal_patch)
    gh, gw = H // patch, W // patch
    out = np.empty((T * gh * gw, C * temporal_patch * patch * patch), dtype=np.float64)
    for t in range(T):
        idx = [min(t * temporal_patch + tt, F - 1) for tt in range(temporal_patch)]
        for h in range(gh):
            for w in range(gw):
                block = frames[idx][:, :, h * patch:(h + 1) * patch, w * patch:(w + 1) * patch]  # [tp, C, p, p]
                out[(t * gh + h) * gw + w] = block.transpose(1, 0, 2, 3).reshape(-1)  # (c, t, kh, kw)
    return out


def patch_embed(patches: np.ndarray, weight: np.ndarray, bias: np.ndarray) -> np.ndarray:
    """Conv3d with kernel = stride = (tp, p, p) as a matrix product (model card,
    Architecture: Conv3d patch embed).  weight is [hidden, 3, tp, p, p]."""
    return patches @ weight.reshape(weight.shape[0], -1).T + bias


# -------------------------------------------------------------- preprocessing

def cubic_kernel(x: float, a: float = -0.5) -> float:
    """Keys' cubic convolution kernel: 1 at 0, 0 at every other integer, support |x| < 2
    (findings section 3 names a bicubic resize; a = -0.5 is the reading)."""
    x = abs(x)
    if x <= 1.0:
        return ((a + 2.0) * x - (a + 3.0)) * x * x + 1.0
    if x < 2.0:
        return (((x - 5.0) * x + 8.0) * x - 4.0) * a
    return 0.0


def resize_taps(n_in: int, n_out: int) -> list[tuple[int, np.ndarray]]:
    """For each output index i along one axis: (first input index, weights summing to 1).

    Output pixel i has its centre at input coordinate c = (i + 1/2) * n_in / n_out (pixel
    centres at half-integers).  When shrinking (n_in > n_out) the kernel is stretched by
    the scale so every input pixel contributes (antialiasing); input pixels j with
    |j + 1/2 - c| inside the support get weight cubic_kernel((j + 1/2 - c) / stretch),
    pixels outside the image are left out and the weights are divided by their sum.
    """
    scale = n_in / n_out
    stretch = max(scale, 1.0)
    support = 2.0 * stretch
    taps = []
    for i in range(n_out):
        c = (i + 0.5) * scale
        lo = max(int(c - support + 0.5), 0)
        hi = min(int(c + support + 0.5), n_in)
        w = np.array([cubic_kernel((j + 0.5 - c) / stretch) for j in range(lo, hi)], dtype=np.float64)
        taps.append((lo, w / w.sum()))
    return taps


def resize_bicubic(img: np.ndarray, out_h: int, out_w: int) -> np.ndarray:
    """An image [H, W, C] resampled to [out_h, out_w, C]: the 1D resampling of
    resize_taps along the width, then along the height (the two commute)."""
    H, W, C = img.shape
    src = img.astype(np.float64)
    tmp = np.empty((H, out_w, C), dtype=np.float64)
    for i, (lo, w) in enumerate(resize_taps(W, out_w)):
        tmp[:, i, :] = np.tensordot(w, src[:, lo:lo + len(w), :], axes=([0], [1]))
    out = np.empty((out_h, out_w, C), dtype=np.float64)
    for i, (lo, w) in enumerate(resize_taps(H, out_h)):
        out[i] = np.tensordot(w, tmp[lo:lo + len(w)], axes=([0], [0]))
    return out


def preprocess(img_u8: np.ndarray, out_h: int, out_w: int, mean, std) -> np.ndarray:
    """A decoded RGB image [H, W, 3] of 8-bit values -> model pixels [3, out_h, out_w]:
    bicubic resize, scale by 1/255, subtract the channel mean, divide by the channel
    standard deviation (findings section 3: bicubic resize, CLIP mean/std)."""
    x = resize_bicubic(img_u8, out_h, out_w) / 255.0
    x = (x - np.asarray(mean, np.float64)) / np.asarray(std, np.float64)
    return np.ascontiguousarray(x.transpose(2, 0, 1))


# ------------------------------------------------------- normalisation, GELU

def layer_norm(x: np.ndarray, gamma: np.ndarray, beta: np.ndarray, eps: float) -> np.ndarray:
    """Affine LayerNorm over the last axis (pre-LN CLIP-style block: norm1 / norm2 in
    the qwen3_vl.rs ViTBlock; model card: CLIP-style ViT)."""
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * gamma + beta


def gelu(x: np.ndarray, tanh_form: bool = True) -> np.ndarray:
    """GELU (model card, Architecture).  tanh form:
    0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))); exact form: x Phi(x)."""
    if tanh_form:
        return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)))
    from math import erf, sqrt
    return x * 0.5 * (1.0 + np.vectorize(erf)(x / sqrt(2.0)))


# ---------------------------------------------------------------------- RoPE

def rope_inv_freq(dim: int, theta: float) -> np.ndarray:
    """inv_freq[k] = theta^(-2k/dim) for k < dim/2 (init.rs, VisionEncoder::new,
    RoPE inverse-frequency table), applied per axis section."""
    k = np.arange(dim // 2, dtype=np.float64)
    return theta ** (-2.0 * k / dim)


def positions_raster(t: int, h: int, w: int) -> np.ndarray:
    """(t, h, w) position of every token in raster order, shape [t*h*w, 3]."""
    tt, hh, ww = np.meshgrid(np.arange(t), np.arange(h), np.arange(w), indexing="ij")
    return np.stack([tt.ravel(), hh.ravel(), ww.ravel()], axis=1).astype(np.int64)


def apply_rope_3d(x: np.ndarray, pos: np.ndarray, sections, theta: float) -> np.ndarray:
    """3D rotary embedding (v2_loaders FINDINGS section 3: rope_mode 3d, theta 10000).

    x: [N, H, D]; pos: [N, 3] integer (t, h, w).  Channels [0, s_t) follow t,
    [s_t, s_t+s_h) follow h, the rest follow w.  In a block of size s starting at
    ``off``, the pair (off+j, off+j+s/2) is the 2-vector (a, b) rotated by the angle
    phi = pos_axis * theta^(-2j/s):  a' = a cos phi - b sin phi,  b' = b cos phi + a sin phi.
    """
    assert sum(sections) == x.shape[-1]
    out = x.copy()
    off = 0
    for axis, s in enumerate(sections):
        half = s // 2
        phi = pos[:, axis:axis + 1].astype(np.float64) * rope_inv_freq(s, theta)[None, :]
        c = np.cos(phi)[:, None, :]
        sn = np.sin(phi)[:, None, :]
        a = x[:, :, off:off + half]
        b = x[:, :, off + half:off + s]
        out[:, :, off:off + half] = a * c - b * sn
        out[:, :, off + half:off + s] = b * c + a * sn
        off += s
    return out


# ----------------------------------------------------------------- attention

def attention_probs(q: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """softmax(q k^T * scale) over keys for one head; q [n, D], k [N, D] -> [n, N]."""
    s = (q @ k.T) * scale
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return p / p.sum(axis=1, keepdims=True)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
              rows=None, row_block: int = 512) -> np.ndarray:
    """Bidirectional multi-head attention: O_h = softmax(q_h k_h^T * scale) v_h.

    init.rs (VisionScratch): the ViT attention is a full [seq, seq] score matrix per
    head followed by a row softmax, i.e. the dense non-causal definition.
    q, k, v: [H, N, D].  Returns [n, H, D] for the query rows ``rows`` (all rows by
    default).  Rows are processed ``row_block`` at a time only to bound memory; each
    row's arithmetic is the definition itself.
    """
    H, N, D = q.shape
    rows = np.arange(N) if rows is None else np.asarray(rows)
    out = np.empty((len(rows), H, v.shape[-1]), dtype=np.float64)
    for h in range(H):
        for s0 in range(0, len(rows), row_block):
            r = rows[s0:s0 + row_block]
            out[s0:s0 + len(r), h] = attention_probs(q[h, r], k[h], scale) @ v[h]
    return out


# --------------------------------------------------------------- tower layer

def tower_layer(x: np.ndarray, w: dict, i: int, cfg: dict, pos: np.ndarray | None) -> np.ndarray:
    """One pre-LN ViT block on one image's tokens x [N, hidden] (qwen3_vl.rs ViTBlock:
    norm1, qkv, proj, norm2, fc1, fc2; model card: CLIP-style, GELU, 3D RoPE).

        x = x + O( MHA( RoPE(q), RoPE(k), v ) ),  [q|k|v] = LN1(x) Wqkv^T + bqkv
        x = x + fc2( GELU( fc1( LN2(x) ) ) )

    q, k, v are the three consecutive ``hidden``-wide column blocks of the qkv output;
    head h is columns [h*D, (h+1)*D) of each.  ``pos`` None means no rotary embedding.
    """
    p = f"layers.{i}."
    N, d = x.shape
    H, D = cfg["heads"], cfg["head_dim"]
    xn = layer_norm(x, w[p + "ln1.weight"], w[p + "ln1.bias"], cfg["ln_eps"])
    qkv = xn @ w[p + "attn.qkv.weight"].T + w[p + "attn.qkv.bias"]
    q = qkv[:, 0 * d:1 * d].reshape(N, H, D)
    k = qkv[:, 1 * d:2 * d].reshape(N, H, D)
    v = qkv[:, 2 * d:3 * d].reshape(N, H, D)
    if pos is not None:
        q = apply_rope_3d(q, pos, cfg["rope_sections"], cfg["rope_theta"])
        k = apply_rope_3d(k, pos, cfg["rope_sections"], cfg["rope_theta"])
    o = attention(q.transpose(1, 0, 2), k.transpose(1, 0, 2), v.transpose(1, 0, 2),
                  1.0 / np.sqrt(D)).reshape(N, d)
    x = x + o @ w[p + "attn.o.weight"].T + w[p + "attn.o.bias"]
    xn = layer_norm(x, w[p + "ln2.weight"], w[p + "ln2.bias"], cfg["ln_eps"])
    hmid = gelu(xn @ w[p + "mlp.fc1.weight"].T + w[p + "mlp.fc1.bias"], cfg["gelu_tanh"])
    return x + hmid @ w[p + "mlp.fc2.weight"].T + w[p + "mlp.fc2.bias"]


def tower_layer_rows(x: np.ndarray, w: dict, i: int, cfg: dict, pos: np.ndarray | None,
                     rows) -> np.ndarray:
    """tower_layer evaluated only at the token rows ``rows`` (same definition: every
    key and value still comes from all tokens).  Used to check large images on a
    sample of outputs."""
    p = f"layers.{i}."
    N, d = x.shape
    H, D = cfg["heads"], cfg["head_dim"]
    rows = np.asarray(rows)
    xn = layer_norm(x, w[p + "ln1.weight"], w[p + "ln1.bias"], cfg["ln_eps"])
    qkv = xn @ w[p + "attn.qkv.weight"].T + w[p + "attn.qkv.bias"]
    q = qkv[:, 0 * d:1 * d].reshape(N, H, D)
    k = qkv[:, 1 * d:2 * d].reshape(N, H, D)
    v = qkv[:, 2 * d:3 * d].reshape(N, H, D)
    if pos is not None:
        q = apply_rope_3d(q[rows], pos[rows], cfg["rope_sections"], cfg["rope_theta"])
        k = apply_rope_3d(k, pos, cfg["rope_sections"], cfg["rope_theta"])
    else:
        q = q[rows]
    o = attention(q.transpose(1, 0, 2), k.transpose(1, 0, 2), v.transpose(1, 0, 2),
                  1.0 / np.sqrt(D)).reshape(len(rows), d)
    xr = x[rows] + o @ w[p + "attn.o.weight"].T + w[p + "attn.o.bias"]
    xn = layer_norm(xr, w[p + "ln2.weight"], w[p + "ln2.bias"], cfg["ln_eps"])
    hmid = gelu(xn @ w[p + "mlp.fc1.weight"].T + w[p + "mlp.fc1.bias"], cfg["gelu_tanh"])
    return xr + hmid @ w[p + "mlp.fc2.weight"].T + w[p + "mlp.fc2.bias"]


# ------------------------------------------------------------------ backward
#
# Reverse-mode derivatives of the forward functions above: each takes the forward's
# inputs and the gradient dy of a scalar loss with respect to the forward's output, and
# returns the gradient with respect to the chosen input (J^T dy).

def layer_norm_backward(x: np.ndarray, gamma: np.ndarray, eps: float, dy: np.ndarray) -> np.ndarray:
    """d loss / d x of layer_norm(x, gamma, beta, eps) over the last axis.
    With xhat = (x - mu) / sigma and g = dy * gamma:
        dx = (g - mean(g) - xhat * mean(g * xhat)) / sigma."""
    mu = x.mean(axis=-1, keepdims=True)
    sigma = np.sqrt(((x - mu) ** 2).mean(axis=-1, keepdims=True) + eps)
    xhat = (x - mu) / sigma
    g = dy * gamma
    return (g - g.mean(axis=-1, keepdims=True) - xhat * (g * xhat).mean(axis=-1, keepdims=True)) / sigma


def gelu_backward(z: np.ndarray, dy: np.ndarray, tanh_form: bool = True) -> np.ndarray:
    """d loss / d z of gelu(z): dy * gelu'(z).  tanh form, u = c (z + 0.044715 z^3):
    gelu' = 0.5 (1 + tanh u) + 0.5 z (1 - tanh^2 u) c (1 + 3 * 0.044715 z^2);
    exact form: gelu' = Phi(z) + z phi(z)."""
    if tanh_form:
        c = np.sqrt(2.0 / np.pi)
        th = np.tanh(c * (z + 0.044715 * z ** 3))
        return dy * (0.5 * (1.0 + th) + 0.5 * z * (1.0 - th ** 2) * c * (1.0 + 3 * 0.044715 * z ** 2))
    from math import erf, sqrt
    cdf = 0.5 * (1.0 + np.vectorize(erf)(z / sqrt(2.0)))
    pdf = np.exp(-0.5 * z ** 2) / np.sqrt(2.0 * np.pi)
    return dy * (cdf + z * pdf)


def rope_3d_backward(dy: np.ndarray, pos: np.ndarray, sections, theta: float) -> np.ndarray:
    """d loss / d x of apply_rope_3d(x, pos): every pair is rotated by phi, a linear
    map whose transpose is the rotation by -phi, i.e. the embedding at position -pos."""
    return apply_rope_3d(dy, -pos, sections, theta)


def attention_backward(q: np.ndarray, k: np.ndarray, v: np.ndarray, do: np.ndarray, scale: float):
    """Gradients of O = softmax(q k^T * scale) v for one head (q [n, D], k, v [N, D],
    do = d loss / d O [n, D]).  With P the probabilities:
        dv = P^T do,   dP = do v^T,   dS = P * (dP - rowsum(P * dP)),
        dq = scale dS k,   dk = scale dS^T q."""
    P = attention_probs(q, k, scale)
    dv = P.T @ do
    dP = do @ v.T
    dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
    return scale * dS @ k, scale * dS.T @ q, dv


def tower_layer_backward(x: np.ndarray, w: dict, i: int, cfg: dict, pos: np.ndarray | None,
                         dy: np.ndarray) -> np.ndarray:
    """d loss / d x of tower_layer(x, w, i, cfg, pos) for one image, given
    dy = d loss / d (layer output).  Recomputes the forward's intermediates, then walks
    the block backwards: MLP branch, LN2, output projection, attention, RoPE, qkv, LN1;
    each residual connection passes its gradient through unchanged."""
    p = f"layers.{i}."
    N, d = x.shape
    H, D = cfg["heads"], cfg["head_dim"]
    # forward, keeping what the backward needs
    xn1 = layer_norm(x, w[p + "ln1.weight"], w[p + "ln1.bias"], cfg["ln_eps"])
    qkv = xn1 @ w[p + "attn.qkv.weight"].T + w[p + "attn.qkv.bias"]
    q = qkv[:, 0 * d:1 * d].reshape(N, H, D)
    k = qkv[:, 1 * d:2 * d].reshape(N, H, D)
    v = qkv[:, 2 * d:3 * d].reshape(N, H, D)
    if pos is not None:
        q = apply_rope_3d(q, pos, cfg["rope_sections"], cfg["rope_theta"])
        k = apply_rope_3d(k, pos, cfg["rope_sections"], cfg["rope_theta"])
    o = attention(q.transpose(1, 0, 2), k.transpose(1, 0, 2), v.transpose(1, 0, 2),
                  1.0 / np.sqrt(D)).reshape(N, d)
    x1 = x + o @ w[p + "attn.o.weight"].T + w[p + "attn.o.bias"]
    xn2 = layer_norm(x1, w[p + "ln2.weight"], w[p + "ln2.bias"], cfg["ln_eps"])
    z = xn2 @ w[p + "mlp.fc1.weight"].T + w[p + "mlp.fc1.bias"]
    # MLP branch: x2 = x1 + gelu(z) W2^T + b2
    dz = gelu_backward(z, dy @ w[p + "mlp.fc2.weight"], cfg["gelu_tanh"])
    dx1 = dy + layer_norm_backward(x1, w[p + "ln2.weight"], cfg["ln_eps"], dz @ w[p + "mlp.fc1.weight"])
    # attention branch: x1 = x + o Wo^T + bo
    do = (dx1 @ w[p + "attn.o.weight"]).reshape(N, H, D)
    dq, dk, dv = (np.empty((N, H, D)) for _ in range(3))
    for h in range(H):
        dq[:, h], dk[:, h], dv[:, h] = attention_backward(q[:, h], k[:, h], v[:, h], do[:, h], 1.0 / np.sqrt(D))
    if pos is not None:
        dq = rope_3d_backward(dq, pos, cfg["rope_sections"], cfg["rope_theta"])
        dk = rope_3d_backward(dk, pos, cfg["rope_sections"], cfg["rope_theta"])
    dqkv = np.concatenate([dq.reshape(N, d), dk.reshape(N, d), dv.reshape(N, d)], axis=1)
    return dx1 + layer_norm_backward(x, w[p + "ln1.weight"], cfg["ln_eps"], dqkv @ w[p + "attn.qkv.weight"])


def patch_fold(du: np.ndarray, H: int, W: int, patch: int = 14, temporal_patch: int = 2) -> np.ndarray:
    """Transpose of patch_unfold: gradients of the patch vectors [gh*gw, 3*tp*p*p]
    (raster) -> gradient of the image [3, H, W].  Each pixel sits in one patch, once per
    repeated frame, so its gradient is the sum over those tp copies."""
    gh, gw = H // patch, W // patch
    out = np.zeros((3, H, W), dtype=np.float64)
    blocks = du.reshape(gh, gw, 3, temporal_patch, patch, patch).sum(axis=3)  # [gh, gw, 3, p, p]
    for h in range(gh):
        for w_ in range(gw):
            out[:, h * patch:(h + 1) * patch, w_ * patch:(w_ + 1) * patch] = blocks[h, w_]
    return out


def tower_backward(pixels: np.ndarray, w: dict, cfg: dict, d_tower: np.ndarray,
                   layers: int | None = None) -> dict:
    """Gradient of a loss with respect to the pixels [B, 3, H, W], given its gradient
    d_tower [B, N, hidden] with respect to the tower output (raster order).  Returns
    dict(tower=the forward's tower output, d_pixels=[B, 3, H, W])."""
    p, tp = cfg["patch"], cfg["temporal_patch"]
    L = cfg["layers"] if layers is None else layers
    tows, grads = [], []
    for b in range(pixels.shape[0]):
        img = pixels[b].astype(np.float64)
        gh, gw = img.shape[1] // p, img.shape[2] // p
        pos = positions_raster(1, gh, gw) if cfg.get("use_rope", True) else None
        xs = [patch_embed(patch_unfold(img, p, tp), w["embeddings.proj.weight"], w["embeddings.proj.bias"])]
        for i in range(L):
            xs.append(tower_layer(xs[-1], w, i, cfg, pos))
        dx = d_tower[b].astype(np.float64)
        for i in reversed(range(L)):
            dx = tower_layer_backward(xs[i], w, i, cfg, pos, dx)
        wpe = w["embeddings.proj.weight"]
        du = dx @ wpe.reshape(wpe.shape[0], -1)
        tows.append(xs[-1])
        grads.append(patch_fold(du, img.shape[1], img.shape[2], p, tp))
    return dict(tower=np.stack(tows), d_pixels=np.stack(grads))


# ------------------------------------------------------- merge and projector

def merge_2x2(x: np.ndarray, t: int, h: int, w: int) -> np.ndarray:
    """2x2 spatial merge (model card: "2x2 spatial merge"; 5120-wide merged tokens are
    2x2 of 1280).  x [t*h*w, C] raster -> [t*(h/2)*(w/2), 4C]; merged (i, j)
    concatenates tokens (2i,2j), (2i,2j+1), (2i+1,2j), (2i+1,2j+1)."""
    C = x.shape[1]
    g = x.reshape(t, h, w, C)
    out = np.empty((t, h // 2, w // 2, 4 * C), dtype=x.dtype)
    for i in range(h // 2):
        for j in range(w // 2):
            out[:, i, j] = np.concatenate(
                [g[:, 2 * i, 2 * j], g[:, 2 * i, 2 * j + 1],
                 g[:, 2 * i + 1, 2 * j], g[:, 2 * i + 1, 2 * j + 1]], axis=-1)
    return out.reshape(t * (h // 2) * (w // 2), 4 * C)


def projector(x: np.ndarray, w: dict, cfg: dict, t: int, h: int, w_: int) -> np.ndarray:
    """Projector (model card, Architecture): Linear(d, P), GELU, Linear(P, P) on every
    tower token; flatten the four P-wide tokens of each 2x2 group (4P wide);
    Linear(4P, P), GELU, Linear(P, P_out)."""
    g = cfg["proj_gelu_tanh"]
    y = gelu(x @ w["proj.patch_fc1.weight"].T + w["proj.patch_fc1.bias"], g)
    y = y @ w["proj.patch_fc2.weight"].T + w["proj.patch_fc2.bias"]
    ym = merge_2x2(y, t, h, w_)
    z = gelu(ym @ w["proj.merge_fc1.weight"].T + w["proj.merge_fc1.bias"], g)
    return z @ w["proj.merge_fc2.weight"].T + w["proj.merge_fc2.bias"]


def projector_rows(x: np.ndarray, w: dict, cfg: dict, t: int, h: int, w_: int,
                   merged_rows) -> np.ndarray:
    """projector evaluated only at the merged tokens ``merged_rows``: each needs just
    the four tower tokens it gathers (merge_source_map)."""
    src = merge_source_map(t, h, w_)[np.asarray(merged_rows)]  # [n, 4]
    g = cfg["proj_gelu_tanh"]
    y = gelu(x[src.ravel()] @ w["proj.patch_fc1.weight"].T + w["proj.patch_fc1.bias"], g)
    y = y @ w["proj.patch_fc2.weight"].T + w["proj.patch_fc2.bias"]
    ym = y.reshape(len(src), -1)
    z = gelu(ym @ w["proj.merge_fc1.weight"].T + w["proj.merge_fc1.bias"], g)
    return z @ w["proj.merge_fc2.weight"].T + w["proj.merge_fc2.bias"]


# ------------------------------------------------------------------- forward

def forward(pixels: np.ndarray, w: dict, cfg: dict, keep_layers: bool = False,
            layers: int | None = None) -> dict:
    """Tower + merge + projector for a batch of images pixels [B, 3, H, W].

    Returns dict(tower=[B, N, d], merged=[B, N/4, 4d], out=[B, N/4, P_out]) and, with
    ``keep_layers``, ``layer_in`` / ``layer_out`` lists of [B, N, d] per layer.
    ``layers`` runs only the first layers (used for bounded CPU timing).
    """
    B = pixels.shape[0]
    p, tp = cfg["patch"], cfg["temporal_patch"]
    L = cfg["layers"] if layers is None else layers
    tows, merged, outs = [], [], []
    lin = [[] for _ in range(L)]
    lout = [[] for _ in range(L)]
    for b in range(B):
        img = pixels[b].astype(np.float64)
        gh, gw = img.shape[1] // p, img.shape[2] // p
        pos = positions_raster(1, gh, gw) if cfg.get("use_rope", True) else None
        x = patch_embed(patch_unfold(img, p, tp), w["embeddings.proj.weight"],
                        w["embeddings.proj.bias"])
        for i in range(L):
            if keep_layers:
                lin[i].append(x)
            x = tower_layer(x, w, i, cfg, pos)
            if keep_layers:
                lout[i].append(x)
        tows.append(x)
        merged.append(merge_2x2(x, 1, gh, gw))
        outs.append(projector(x, w, cfg, 1, gh, gw))
    res = dict(tower=np.stack(tows), merged=np.stack(merged), out=np.stack(outs))
    if keep_layers:
        res["layer_in"] = [np.stack(a) for a in lin]
        res["layer_out"] = [np.stack(a) for a in lout]
    return res


def forward_video(clips: np.ndarray, w: dict, cfg: dict, layers: int | None = None) -> dict:
    """Tower + merge + projector for clips [B, F, 3, H, W]: T = ceil(F/tp) temporal
    patches, all T*gh*gw tokens of a clip attend to each other, RoPE positions
    (t, h, w), the 2x2 merge within each temporal slice."""
    p, tp = cfg["patch"], cfg["temporal_patch"]
    L = cfg["layers"] if layers is None else layers
    tows, outs = [], []
    for b in range(clips.shape[0]):
        clip = clips[b].astype(np.float64)
        T = -(-clip.shape[0] // tp)
        gh, gw = clip.shape[2] // p, clip.shape[3] // p
        pos = positions_raster(T, gh, gw) if cfg.get("use_rope", True) else None
        x = patch_embed(patch_unfold_video(clip, p, tp), w["embeddings.proj.weight"], w["embeddings.proj.bias"])
        for i in range(L):
            x = tower_layer(x, w, i, cfg, pos)
        tows.append(x)
        outs.append(projector(x, w, cfg, T, gh, gw))
    return dict(tower=np.stack(tows), out=np.stack(outs))


# ----------------------------------------------------------------- index maps

def block_order(t: int, h: int, w: int) -> np.ndarray:
    """Raster index of the token at each position of 2x2-block order: the four tokens
    of merged group (i, j) are consecutive, in the merge's member order, and the groups
    follow raster (i, j) order.  Used only to compare index maps exactly."""
    out = []
    for tt in range(t):
        for i in range(h // 2):
            for j in range(w // 2):
                for di in (0, 1):
                    for dj in (0, 1):
                        out.append(tt * h * w + (2 * i + di) * w + (2 * j + dj))
    return np.asarray(out, dtype=np.int64)


def merge_source_map(t: int, h: int, w: int) -> np.ndarray:
    """[t*(h/2)*(w/2), 4] raster indices of the four tokens each merged token gathers."""
    idx = np.arange(t * h * w, dtype=np.int64)[:, None]
    return merge_2x2(idx, t, h, w).astype(np.int64)
