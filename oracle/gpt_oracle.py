"""Oracle: a plain, slow CPU implementation of one GPT training step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The product library never calls it, and it imports nothing from the
product package: the two share no code.  The only thing both sides consume is
the seeded input generator in ``scratch_decoder_only_b200.synthetic``, which
holds none of the method's arithmetic.

What it computes, with the page each step follows:

* token embedding plus a learned position embedding, added directly --
  "Feste: GPT-2 from scratch in Rust", section "Model Architecture mirrors
  GPT-2" (embeddings with positional encoding added);
* pre-LayerNorm blocks: LN -> causal multi-head attention -> residual,
  LN -> GELU MLP -> residual; a final LN after the last block -- same section,
  and "LucilleAI", section "Architecture (from source)" (block/stack,
  attention, FFN, LayerNorm);
* causal masking by setting future scores to -inf before the softmax
  (masked_fill) -- Feste, same section; packed sequences attend only inside
  their own document -- LucilleAI, sections "What makes it special" and
  "Real measured numbers" (sequence packing);
* the output projection to the vocabulary -- "RustGPT", section "Key files"
  (output_projection.rs);
* softmax cross-entropy on the next token -- RustGPT, section "Technical
  implementation" (cross-entropy loss); Smallem, "Ce qu'est un modele de
  langage" (train = raise the probability of the true next token);
* a hand-written backward pass by the chain rule through softmax, the heads
  and the residuals -- Feste, section "Manual Backpropagation from scratch";
* global L2 gradient clipping -- RustGPT, "Technical implementation" (L2 norm
  capped at 5.0); AdamW with decoupled weight decay -- Feste, same backprop
  section;
* dynamic loss scaling with skip-on-overflow -- LucilleAI, "Architecture"
  (GradScaler, AMP);
* greedy decoding: take the argmax, append it, repeat -- RustGPT "Technical
  implementation" (greedy decoding); Smallem "Ce qu'est un modele de langage";
* sampled decoding (temperature, top-k, top-p) and beam search -- RustGPT,
  roadmap "high-priority feature requests" (better sampling); the learning-rate
  schedule -- LucilleAI, "Getting started" (cosine, warm-up, min-lr); the
  Llama-style block (RMSNorm, rotary positions, grouped key/value heads,
  SwiGLU) -- "NTransformer", key features.

Where the pages leave a step open the plainest reading is taken (GPT-2's
LayerNorm eps 1e-5 with biased variance, tanh-form GELU, biases on every
linear layer except the LM head, scale 1/sqrt(d), loss averaged over valid
targets, weight decay on every parameter, PyTorch clip semantics
coef = min(1, c / (norm + 1e-6))).

Floating point: every function takes ``dtype`` (float64 by default; float32
where a decision must be taken in the kernel's precision, e.g. the greedy
argmax).  numpy's matmul is used as the contraction primitive; there is no
blocking, fusion or reordering beyond the definitions below.

Parity status: every function in this module is pinned by
``tests/test_oracle_pins.py`` (finite differences over every parameter
element, closed forms, invariants, published test vectors).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

GELU_K = math.sqrt(2.0 / math.pi)
GELU_C = 0.044715


@dataclass(frozen=True)
class OracleConfig:
    vocab: int
    vocab_padded: int
    d_model: int
    n_heads: int
    d_mlp: int
    n_layers: int
    max_seq: int
    tied: bool = False
    ln_eps: float = 1e-5
    init_std: float = 0.02
    arch: str = "gpt2"          # "gpt2" or "llama"
    n_kv_heads: int = 0         # llama: key / value heads (0: n_heads)
    rope_base: float = 10000.0  # llama: rotary base

    @property
    def head_dim(self) -> int:
        return self.d_model // self.n_heads

    @property
    def kv_heads(self) -> int:
        return self.n_kv_heads or self.n_heads


# ---------------------------------------------------------------------------
# Parameters: canonical order and initialisation
# ---------------------------------------------------------------------------

def param_shapes(cfg: OracleConfig):
    """Canonical parameter order (row-major, linear weights stored [out, in])."""
    C, F, Vp = cfg.d_model, cfg.d_mlp, cfg.vocab_padded
    if cfg.arch == "llama":
        # no position table, no biases; q rows, then the key heads', then the
        # value heads' rows; gate rows, then up rows
        kvd = cfg.kv_heads * cfg.head_dim
        out = [("wte", (Vp, C))]
        for l in range(cfg.n_layers):
            p = f"h{l}."
            out += [(p + "attn_norm_g", (C,)), (p + "w_qkv", (C + 2 * kvd, C)), (p + "w_o", (C, C)),
                    (p + "mlp_norm_g", (C,)), (p + "w_gu", (2 * F, C)), (p + "w_down", (C, F))]
        out += [("norm_g", (C,))]
        if not cfg.tied:
            out.append(("w_head", (Vp, C)))
        return out
    out = [("wte", (Vp, C)), ("wpe", (cfg.max_seq, C))]
    for l in range(cfg.n_layers):
        p = f"h{l}."
        out += [
            (p + "ln1_g", (C,)), (p + "ln1_b", (C,)),
            (p + "w_qkv", (3 * C, C)), (p + "b_qkv", (3 * C,)),
            (p + "w_o", (C, C)), (p + "b_o", (C,)),
            (p + "ln2_g", (C,)), (p + "ln2_b", (C,)),
            (p + "w_fc", (F, C)), (p + "b_fc", (F,)),
            (p + "w_fc2", (C, F)), (p + "b_fc2", (C,)),
        ]
    out += [("lnf_g", (C,)), ("lnf_b", (C,))]
    if not cfg.tied:
        out.append(("w_head", (Vp, C)))
    return out


def num_params(cfg: OracleConfig) -> int:
    return sum(int(np.prod(s)) for _, s in param_shapes(cfg))


def unflatten(cfg: OracleConfig, flat: np.ndarray) -> dict:
    """Views into ``flat`` by name; ``w_head`` aliases ``wte`` when tied."""
    views, o = {}, 0
    for name, shape in param_shapes(cfg):
        n = int(np.prod(shape))
        views[name] = flat[o:o + n].reshape(shape)
        o += n
    assert o == flat.size
    if cfg.tied:
        views["w_head"] = views["wte"]
    return views


_SM64_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_SM64_M1 = np.uint64(0xBF58476D1CE4E5B9)
_SM64_M2 = np.uint64(0x94D049BB133111EB)


def splitmix64(seed: int, counters: np.ndarray) -> np.ndarray:
    """SplitMix64 output number ``k`` (0-based) for every k in ``counters``.

    Steele, Lea and Flood, "Fast splittable pseudorandom number generators"
    (OOPSLA 2014), in the form of Vigna's reference splitmix64.c: the state is
    advanced by the golden-ratio increment and each output is the state after
    k+1 increments passed through the variant-13 finaliser.  Computed in
    wrapping uint64 arithmetic.
    """
    with np.errstate(over="ignore"):
        k = counters.astype(np.uint64)
        z = np.uint64(seed) + (k + np.uint64(1)) * _SM64_GAMMA
        z = (z ^ (z >> np.uint64(30))) * _SM64_M1
        z = (z ^ (z >> np.uint64(27))) * _SM64_M2
        return z ^ (z >> np.uint64(31))


def gaussian_for_elements(seed: int, elem: np.ndarray) -> np.ndarray:
    """Standard normal deviate for canonical element index ``e`` (float64).

    Box and Muller (1958): draws 2e and 2e+1 of the SplitMix64 stream give
    u1 = ((x >> 11) + 1) * 2^-53 in (0, 1] and u2 = (x >> 11) * 2^-53 in [0, 1);
    z = sqrt(-2 ln u1) * cos(2 pi u2).
    """
    e = elem.astype(np.uint64)
    x1 = splitmix64(seed, np.uint64(2) * e)
    x2 = splitmix64(seed, np.uint64(2) * e + np.uint64(1))
    u1 = ((x1 >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)
    u2 = (x2 >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


def init_params(cfg: OracleConfig, seed: int) -> np.ndarray:
    """Initial fp32 parameter vector in canonical order.

    Weight matrices and embeddings ~ N(0, init_std) (value for canonical
    element e: float32(std * gaussian_for_elements(seed, e)) with std the
    float32 value of init_std), LayerNorm gains 1,
    LayerNorm shifts and biases 0, and the padded vocabulary rows V..Vp-1 of
    the embedding / LM head are 0.
    """
    flat = np.zeros(num_params(cfg), dtype=np.float32)
    # the configured standard deviation at float32 precision, as a
    # configuration record carries it (0.02 -> 0.0199999995529651...)
    std = float(np.float32(cfg.init_std))
    o = 0
    for name, shape in param_shapes(cfg):
        n = int(np.prod(shape))
        leaf = name.split(".")[-1]
        if leaf in ("wte", "wpe", "w_qkv", "w_o", "w_fc", "w_fc2", "w_head", "w_gu", "w_down"):
            z = gaussian_for_elements(seed, np.arange(o, o + n, dtype=np.uint64))
            vals = (std * z).astype(np.float32)
            if leaf in ("wte", "w_head"):
                vals.reshape(shape)[cfg.vocab:, :] = 0.0
            flat[o:o + n] = vals
        elif leaf.endswith("_g"):
            flat[o:o + n] = 1.0
        o += n
    return flat


# ---------------------------------------------------------------------------
# Elementary pieces (each pinned on its own)
# ---------------------------------------------------------------------------

def positions_from_segments(seg_ids: np.ndarray | None, B: int, T: int):
    """Position of every token inside its document, and the document id.

    Without seg_ids every row is one document and pos = t.  With seg_ids
    (documents are contiguous runs inside a row) the position restarts at 0
    at the first token of every run.
    """
    if seg_ids is None:
        seg = np.zeros((B, T), dtype=np.int64)
    else:
        seg = np.asarray(seg_ids, dtype=np.int64).reshape(B, T)
    pos = np.zeros((B, T), dtype=np.int64)
    for b in range(B):
        for t in range(1, T):
            pos[b, t] = pos[b, t - 1] + 1 if seg[b, t] == seg[b, t - 1] else 0
    return pos, seg


def layernorm_fwd(x, g, b, eps):
    """(x - mean) / sqrt(var + eps) * g + b over the last axis, biased var."""
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + eps)
    xhat = (x - mu) * rstd
    return xhat * g + b, xhat, rstd


def layernorm_bwd(dy, xhat, rstd, g):
    """Chain rule through LayerNorm: returns dx, dg, db (dg, db summed over rows)."""
    gh = dy * g
    C = xhat.shape[-1]
    dx = rstd * (gh - gh.sum(-1, keepdims=True) / C
                 - xhat * (gh * xhat).sum(-1, keepdims=True) / C)
    dg = (dy * xhat).reshape(-1, C).sum(0)
    db = dy.reshape(-1, C).sum(0)
    return dx, dg, db


def gelu(u):
    """GELU in GPT-2's tanh form: 0.5 u (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3)))."""
    return 0.5 * u * (1.0 + np.tanh(GELU_K * (u + GELU_C * u ** 3)))


def gelu_grad(u):
    """d gelu / du for the tanh form above."""
    t = np.tanh(GELU_K * (u + GELU_C * u ** 3))
    return 0.5 * (1.0 + t) + 0.5 * u * (1.0 - t * t) * GELU_K * (1.0 + 3.0 * GELU_C * u * u)


def allowed_mask(seg_row: np.ndarray) -> np.ndarray:
    """allowed[i, j]: key j is visible to query i (j <= i, same document)."""
    T = seg_row.shape[0]
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    return (j <= i) & (seg_row[None, :] == seg_row[:, None])


def softmax_rows(s):
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def attention_probs(q, k, allowed):
    """P = softmax(q k^T / sqrt(d)) with disallowed scores set to -inf first.

    q, k: [H, T, d] for one batch row; allowed: [T, T].
    """
    d = q.shape[-1]
    s = (q @ np.swapaxes(k, -1, -2)) * (1.0 / math.sqrt(d))
    s = np.where(allowed[None], s, -np.inf)
    return softmax_rows(s)


def attention_fwd(q, k, v, seg):
    """o = P v per (batch row, head); q, k, v: [B, H, T, d]."""
    o = np.empty_like(q)
    for b in range(q.shape[0]):
        p = attention_probs(q[b], k[b], allowed_mask(seg[b]))
        o[b] = p @ v[b]
    return o


def attention_bwd(q, k, v, seg, do):
    """Chain rule through o = softmax(q k^T / sqrt(d)) v, P recomputed."""
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    scale = 1.0 / math.sqrt(q.shape[-1])
    for b in range(q.shape[0]):
        p = attention_probs(q[b], k[b], allowed_mask(seg[b]))
        dv[b] = np.swapaxes(p, -1, -2) @ do[b]
        dp = do[b] @ np.swapaxes(v[b], -1, -2)
        ds = p * (dp - (dp * p).sum(-1, keepdims=True))
        dq[b] = (ds @ k[b]) * scale
        dk[b] = (np.swapaxes(ds, -1, -2) @ q[b]) * scale
    return dq, dk, dv


def cross_entropy(z, targets, V):
    """Mean over valid targets (>= 0) of logsumexp(z[:V]) - z[target].

    Returns (loss, dz) where dz = (softmax - onehot) / N_valid on the first V
    columns of valid rows and 0 elsewhere (padded columns, ignored rows).
    """
    zv = z[:, :V]
    m = zv.max(axis=1, keepdims=True)
    e = np.exp(zv - m)
    ssum = e.sum(axis=1, keepdims=True)
    lse = (m + np.log(ssum))[:, 0]
    valid = targets >= 0
    n_valid = int(valid.sum())
    rows = np.nonzero(valid)[0]
    tgt = targets[rows]
    loss = float((lse[rows] - zv[rows, tgt]).sum() / n_valid) if n_valid else 0.0
    dz = np.zeros_like(z)
    if n_valid:
        dz[rows, :V] = e[rows] / ssum[rows]
        dz[rows, tgt] -= 1.0
        dz /= n_valid
    return loss, dz


# ---------------------------------------------------------------------------
# Model forward / backward
# ---------------------------------------------------------------------------

def _split_heads(x, B, T, H, d):
    return x.reshape(B, T, H, d).transpose(0, 2, 1, 3)


def _merge_heads(x, B, T, H, d):
    return x.transpose(0, 2, 1, 3).reshape(B * T, H * d)


def forward(cfg: OracleConfig, flat_params, tokens, seg_ids=None, dtype=np.float64):
    """Logits [B*T, Vp] and the cache the backward pass needs."""
    if cfg.arch == "llama":
        return forward_llama(cfg, flat_params, tokens, seg_ids, dtype)
    P = {k: v.astype(dtype) for k, v in unflatten(cfg, np.asarray(flat_params)).items()}
    tokens = np.asarray(tokens, dtype=np.int64)
    B, T = tokens.shape
    C, H, d = cfg.d_model, cfg.n_heads, cfg.head_dim
    pos, seg = positions_from_segments(seg_ids, B, T)
    x = P["wte"][tokens.reshape(-1)] + P["wpe"][pos.reshape(-1)]
    cache = dict(B=B, T=T, tokens=tokens, pos=pos, seg=seg, layers=[], P=P)
    for l in range(cfg.n_layers):
        p = f"h{l}."
        lc = {"x_in": x}
        h1, lc["xhat1"], lc["rstd1"] = layernorm_fwd(x, P[p + "ln1_g"], P[p + "ln1_b"], cfg.ln_eps)
        lc["h1"] = h1
        qkv = h1 @ P[p + "w_qkv"].T + P[p + "b_qkv"]
        q = _split_heads(qkv[:, :C], B, T, H, d)
        k = _split_heads(qkv[:, C:2 * C], B, T, H, d)
        v = _split_heads(qkv[:, 2 * C:], B, T, H, d)
        lc["q"], lc["k"], lc["v"] = q, k, v
        o = _merge_heads(attention_fwd(q, k, v, seg), B, T, H, d)
        lc["o"] = o
        x = x + o @ P[p + "w_o"].T + P[p + "b_o"]
        lc["x_mid"] = x
        h2, lc["xhat2"], lc["rstd2"] = layernorm_fwd(x, P[p + "ln2_g"], P[p + "ln2_b"], cfg.ln_eps)
        lc["h2"] = h2
        u = h2 @ P[p + "w_fc"].T + P[p + "b_fc"]
        a = gelu(u)
        lc["u"], lc["a"] = u, a
        x = x + a @ P[p + "w_fc2"].T + P[p + "b_fc2"]
        cache["layers"].append(lc)
    xf, cache["xhatf"], cache["rstdf"] = layernorm_fwd(x, P["lnf_g"], P["lnf_b"], cfg.ln_eps)
    cache["xf"] = xf
    logits = xf @ P["w_head"].T
    return logits, cache


def backward(cfg: OracleConfig, cache, dlogits):
    """Gradients of every parameter (dict by name, untied names only)."""
    if cfg.arch == "llama":
        return backward_llama(cfg, cache, dlogits)
    P = cache["P"]
    B, T = cache["B"], cache["T"]
    C, H, d = cfg.d_model, cfg.n_heads, cfg.head_dim
    G = {}
    g_head = dlogits.T @ cache["xf"]
    dxf = dlogits @ P["w_head"]
    dx, G["lnf_g"], G["lnf_b"] = layernorm_bwd(dxf, cache["xhatf"], cache["rstdf"], P["lnf_g"])
    for l in reversed(range(cfg.n_layers)):
        p = f"h{l}."
        lc = cache["layers"][l]
        # MLP branch: x_out = x_mid + gelu(LN2(x_mid) W_fc^T + b_fc) W_fc2^T + b_fc2
        G[p + "b_fc2"] = dx.sum(0)
        G[p + "w_fc2"] = dx.T @ lc["a"]
        da = dx @ P[p + "w_fc2"]
        du = da * gelu_grad(lc["u"])
        G[p + "b_fc"] = du.sum(0)
        G[p + "w_fc"] = du.T @ lc["h2"]
        dh2 = du @ P[p + "w_fc"]
        dln, G[p + "ln2_g"], G[p + "ln2_b"] = layernorm_bwd(dh2, lc["xhat2"], lc["rstd2"], P[p + "ln2_g"])
        dx = dx + dln
        # attention branch: x_mid = x_in + attn(LN1(x_in)) W_o^T + b_o
        G[p + "b_o"] = dx.sum(0)
        G[p + "w_o"] = dx.T @ lc["o"]
        do = _split_heads(dx @ P[p + "w_o"], B, T, H, d)
        dq, dk, dv = attention_bwd(lc["q"], lc["k"], lc["v"], cache["seg"], do)
        dqkv = np.concatenate([_merge_heads(t, B, T, H, d) for t in (dq, dk, dv)], axis=1)
        G[p + "b_qkv"] = dqkv.sum(0)
        G[p + "w_qkv"] = dqkv.T @ lc["h1"]
        dh1 = dqkv @ P[p + "w_qkv"]
        dln, G[p + "ln1_g"], G[p + "ln1_b"] = layernorm_bwd(dh1, lc["xhat1"], lc["rstd1"], P[p + "ln1_g"])
        dx = dx + dln
    # embeddings: scatter-add of the residual gradient by token and by position
    g_wte = np.zeros_like(P["wte"])
    np.add.at(g_wte, cache["tokens"].reshape(-1), dx)
    g_wpe = np.zeros_like(P["wpe"])
    np.add.at(g_wpe, cache["pos"].reshape(-1), dx)
    if cfg.tied:
        G["wte"] = g_wte + g_head
    else:
        G["wte"] = g_wte
        G["w_head"] = g_head
    G["wpe"] = g_wpe
    return G


# ---------------------------------------------------------------------------
# Llama-style block: RMSNorm, rotary positions, grouped key / value heads,
# SwiGLU MLP ("NTransformer" page, key features: Llama architecture with RoPE,
# GQA and SwiGLU, KV cache; "RustGPT" roadmap: architecture extensions)
# ---------------------------------------------------------------------------

def rmsnorm_fwd(x, g, eps):
    """x / sqrt(mean(x^2) + eps) * g over the last axis (Zhang and Sennrich 2019)."""
    rstd = 1.0 / np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps)
    xhat = x * rstd
    return xhat * g, xhat, rstd


def rmsnorm_bwd(dy, xhat, rstd, g):
    """Chain rule through RMSNorm: returns dx, dg (dg summed over rows)."""
    gh = dy * g
    C = xhat.shape[-1]
    dx = rstd * (gh - xhat * (gh * xhat).sum(-1, keepdims=True) / C)
    dg = (dy * xhat).reshape(-1, C).sum(0)
    return dx, dg


def rope_angles(pos, d, base):
    """Angle pos * theta_i of dimension pair i = 0..d/2-1, theta_i = base^(-2i/d)
    (Su et al., RoFormer), for positions pos [B, T] -> [B, T, d/2]."""
    i = np.arange(d // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / d)
    return np.asarray(pos, dtype=np.float64)[..., None] * theta


def rope_apply(x, ang, inverse=False):
    """Rotate the consecutive pairs (x[2i], x[2i+1]) of the last axis by ang
    (or by -ang: the transpose, for the backward pass).  x: [B, H, T, d],
    ang: [B, T, d/2]."""
    c = np.cos(ang)[:, None]
    s = np.sin(ang)[:, None]
    if inverse:
        s = -s
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


def silu(z):
    return z / (1.0 + np.exp(-z))


def silu_grad(z):
    sg = 1.0 / (1.0 + np.exp(-z))
    return sg * (1.0 + z * (1.0 - sg))


def _expand_kv(x, G):
    """[B, Hkv, T, d] -> [B, Hkv * G, T, d]: query head h reads key head h // G."""
    return np.repeat(x, G, axis=1)


def forward_llama(cfg: OracleConfig, flat_params, tokens, seg_ids=None, dtype=np.float64):
    """Logits [B*T, Vp] of the Llama-style model and the backward cache.

    Block: h = RMSNorm(x) g1; q, k, v = h W_qkv^T (H query heads, Hkv key /
    value heads); q, k rotated by their position inside the document; causal
    (block-diagonal when packed) attention with query head h on key / value
    head h // (H / Hkv); x += o W_o^T; h2 = RMSNorm(x) g2; gate, up = h2
    W_gu^T; x += (silu(gate) * up) W_down^T.  Then RMSNorm and the head.
    """
    P = {k: v.astype(dtype) for k, v in unflatten(cfg, np.asarray(flat_params)).items()}
    tokens = np.asarray(tokens, dtype=np.int64)
    B, T = tokens.shape
    C, H, d, F = cfg.d_model, cfg.n_heads, cfg.head_dim, cfg.d_mlp
    Hkv = cfg.kv_heads
    G = H // Hkv
    pos, seg = positions_from_segments(seg_ids, B, T)
    ang = rope_angles(pos, d, cfg.rope_base)
    x = P["wte"][tokens.reshape(-1)]
    cache = dict(B=B, T=T, tokens=tokens, pos=pos, seg=seg, ang=ang, layers=[], P=P)
    for l in range(cfg.n_layers):
        p = f"h{l}."
        lc = {}
        h1, lc["xhat1"], lc["rstd1"] = rmsnorm_fwd(x, P[p + "attn_norm_g"], cfg.ln_eps)
        lc["h1"] = h1
        qkv = h1 @ P[p + "w_qkv"].T
        q = rope_apply(_split_heads(qkv[:, :C], B, T, H, d), ang)
        k = rope_apply(_split_heads(qkv[:, C:C + Hkv * d], B, T, Hkv, d), ang)
        v = _split_heads(qkv[:, C + Hkv * d:], B, T, Hkv, d)
        lc["q"], lc["k"], lc["v"] = q, k, v
        o = _merge_heads(attention_fwd(q, _expand_kv(k, G), _expand_kv(v, G), seg), B, T, H, d)
        lc["o"] = o
        x = x + o @ P[p + "w_o"].T
        h2, lc["xhat2"], lc["rstd2"] = rmsnorm_fwd(x, P[p + "mlp_norm_g"], cfg.ln_eps)
        lc["h2"] = h2
        gu = h2 @ P[p + "w_gu"].T
        lc["gate"], lc["up"] = gu[:, :F], gu[:, F:]
        a = silu(lc["gate"]) * lc["up"]
        lc["a"] = a
        x = x + a @ P[p + "w_down"].T
        cache["layers"].append(lc)
    xf, cache["xhatf"], cache["rstdf"] = rmsnorm_fwd(x, P["norm_g"], cfg.ln_eps)
    cache["xf"] = xf
    return xf @ P["w_head"].T, cache


def backward_llama(cfg: OracleConfig, cache, dlogits):
    """Gradients of every parameter of the Llama-style model (by name)."""
    P = cache["P"]
    B, T, ang = cache["B"], cache["T"], cache["ang"]
    C, H, d, F = cfg.d_model, cfg.n_heads, cfg.head_dim, cfg.d_mlp
    Hkv = cfg.kv_heads
    G = H // Hkv
    Gr = {}
    g_head = dlogits.T @ cache["xf"]
    dxf = dlogits @ P["w_head"]
    dx, Gr["norm_g"] = rmsnorm_bwd(dxf, cache["xhatf"], cache["rstdf"], P["norm_g"])
    for l in reversed(range(cfg.n_layers)):
        p = f"h{l}."
        lc = cache["layers"][l]
        # MLP: x_out = x_mid + (silu(gate) * up) W_down^T
        Gr[p + "w_down"] = dx.T @ lc["a"]
        da = dx @ P[p + "w_down"]
        dgate = da * lc["up"] * silu_grad(lc["gate"])
        dup = da * silu(lc["gate"])
        dgu = np.concatenate([dgate, dup], axis=1)
        Gr[p + "w_gu"] = dgu.T @ lc["h2"]
        dh2 = dgu @ P[p + "w_gu"]
        dln, Gr[p + "mlp_norm_g"] = rmsnorm_bwd(dh2, lc["xhat2"], lc["rstd2"], P[p + "mlp_norm_g"])
        dx = dx + dln
        # attention: x_mid = x_in + attn(RMSNorm(x_in)) W_o^T
        Gr[p + "w_o"] = dx.T @ lc["o"]
        do = _split_heads(dx @ P[p + "w_o"], B, T, H, d)
        dq, dke, dve = attention_bwd(lc["q"], _expand_kv(lc["k"], G), _expand_kv(lc["v"], G), cache["seg"], do)
        # a key / value head's gradient sums over the query heads that read it
        dk = dke.reshape(B, Hkv, G, T, d).sum(axis=2)
        dv = dve.reshape(B, Hkv, G, T, d).sum(axis=2)
        dq = rope_apply(dq, ang, inverse=True)
        dk = rope_apply(dk, ang, inverse=True)
        dqkv = np.concatenate([_merge_heads(dq, B, T, H, d), _merge_heads(dk, B, T, Hkv, d),
                               _merge_heads(dv, B, T, Hkv, d)], axis=1)
        Gr[p + "w_qkv"] = dqkv.T @ lc["h1"]
        dh1 = dqkv @ P[p + "w_qkv"]
        dln, Gr[p + "attn_norm_g"] = rmsnorm_bwd(dh1, lc["xhat1"], lc["rstd1"], P[p + "attn_norm_g"])
        dx = dx + dln
    g_wte = np.zeros_like(P["wte"])
    np.add.at(g_wte, cache["tokens"].reshape(-1), dx)
    if cfg.tied:
        Gr["wte"] = g_wte + g_head
    else:
        Gr["wte"] = g_wte
        Gr["w_head"] = g_head
    return Gr


def flatten_grads(cfg: OracleConfig, G: dict, dtype=np.float64) -> np.ndarray:
    return np.concatenate([np.asarray(G[name], dtype=dtype).reshape(-1)
                           for name, _ in param_shapes(cfg)])


def loss_and_grads(cfg: OracleConfig, flat_params, tokens, targets, seg_ids=None, dtype=np.float64):
    """Forward, softmax cross-entropy and backward: (loss, flat grads)."""
    logits, cache = forward(cfg, flat_params, tokens, seg_ids, dtype)
    loss, dz = cross_entropy(logits, np.asarray(targets).reshape(-1), cfg.vocab)
    G = backward(cfg, cache, dz)
    return loss, flatten_grads(cfg, G, dtype)


# ---------------------------------------------------------------------------
# Optimiser: global clip, AdamW, dynamic loss scale
# ---------------------------------------------------------------------------

def clip_coefficient(grads, clip_norm):
    """coef = min(1, c / (||g||_2 + 1e-6)) over all elements; returns (norm, coef)."""
    norm = float(np.sqrt(np.sum(np.asarray(grads, dtype=np.float64) ** 2)))
    return norm, min(1.0, clip_norm / (norm + 1e-6))


def adamw_update(p, g, m, v, t, lr, beta1, beta2, eps, wd):
    """One AdamW step (t starts at 1) with decoupled weight decay.

    m <- b1 m + (1-b1) g;  v <- b2 v + (1-b2) g^2;
    p <- p - lr (m/(1-b1^t) / (sqrt(v/(1-b2^t)) + eps) + wd p).
    """
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    mhat = m / (1.0 - beta1 ** t)
    vhat = v / (1.0 - beta2 ** t)
    p = p - lr * (mhat / (np.sqrt(vhat) + eps) + wd * p)
    return p, m, v


def loss_scale_update(scale, good_steps, finite, growth_interval=2000):
    """GradScaler's rule: halve and skip on a non-finite step, double after
    ``growth_interval`` consecutive finite steps.  Returns (scale, good, skip)."""
    if not finite:
        return scale * 0.5, 0, True
    good_steps += 1
    if good_steps >= growth_interval:
        return scale * 2.0, 0, False
    return scale, good_steps, False


def lr_at(step, kind, warmup, total, max_lr, min_lr, lr_const=0.0):
    """Learning rate of the AdamW step that follows ``step`` taken steps.

    The pages' SFT recipe uses a cosine schedule with warm-up steps and a
    minimum learning rate ("LucilleAI", "Getting started": --lr-scheduler
    cosine --warmup-steps 100 --min-lr 0.00003).  Read plainly: a linear ramp
    to max_lr over the warm-up steps, then half a cosine period from max_lr
    down to min_lr at step ``total``, then min_lr.  kind 0 = constant.
    """
    if kind == 0:
        return lr_const
    if step < warmup:
        return max_lr * (step + 1) / warmup
    if step >= total:
        return min_lr
    r = (step - warmup) / (total - warmup)
    return min_lr + 0.5 * (max_lr - min_lr) * (1.0 + math.cos(math.pi * r))


def clip_adamw_step(params, grads, m, v, t, lr, beta1, beta2, eps, wd, clip_norm):
    """Clip by the global L2 norm, then AdamW.  Skips (no change) when the
    gradient is not finite.  Returns (p, m, v, norm, skipped)."""
    g = np.asarray(grads, dtype=np.float64)
    norm, coef = clip_coefficient(g, clip_norm)
    if not math.isfinite(norm):
        return params, m, v, norm, True
    p, m2, v2 = adamw_update(np.asarray(params, np.float64), g * coef,
                             np.asarray(m, np.float64), np.asarray(v, np.float64),
                             t, lr, beta1, beta2, eps, wd)
    return p, m2, v2, norm, False


# ---------------------------------------------------------------------------
# Greedy decoding
# ---------------------------------------------------------------------------

def greedy_decode(cfg: OracleConfig, flat_params, prompt, n_new, dtype=np.float32):
    """Greedy continuation by full-prefix recomputation (no cache).

    Each step runs the forward pass over the whole prefix, takes the argmax of
    the last position's logits over the real vocabulary (first index on ties),
    and appends it.  Returns (tokens [B, n_new], top-2 logit gaps [B, n_new]).
    """
    seq = np.asarray(prompt, dtype=np.int64)
    B = seq.shape[0]
    out = np.zeros((B, n_new), dtype=np.int64)
    gaps = np.zeros((B, n_new), dtype=np.float64)
    for s in range(n_new):
        logits, _ = forward(cfg, flat_params, seq, None, dtype)
        last = logits.reshape(B, seq.shape[1], -1)[:, -1, :cfg.vocab]
        nxt = np.argmax(last, axis=1)
        srt = np.sort(last, axis=1)
        gaps[:, s] = srt[:, -1] - srt[:, -2]
        out[:, s] = nxt
        seq = np.concatenate([seq, nxt[:, None]], axis=1)
    return out, gaps


# ---------------------------------------------------------------------------
# Sampling decode: temperature, top-k, top-p
# ---------------------------------------------------------------------------

def sample_token(z, V, temperature, top_k, top_p, u):
    """One sampled token from a row of logits ``z`` (real vocabulary 0..V-1).

    The pages list temperature scaling, top-k and top-p among the generation
    features a from-scratch model should gain after greedy decoding
    ("RustGPT", roadmap "high-priority feature requests"; "LucilleAI" names a
    sampler in its GPU stack).  Read plainly, in this order:

    * temperature <= 0: greedy (argmax, lowest index on ties);
    * x = z / temperature;
    * top-k (0 < top_k < V): keep the top_k largest x, ties at the cut going
      to the lower indices;
    * weights w_i = exp(x_i - max x) over the kept tokens;
    * top-p (top_p < 1): order the kept tokens by (w descending, index
      ascending) and keep the shortest prefix whose weight reaches top_p times
      the kept total (ties at the cut again to the lower indices);
    * with the uniform draw u in [0, 1) (an input: the method's random
      numbers are passed in), return the first kept token, in ascending token
      order, at which the running sum of kept weights exceeds u times their
      total.
    """
    z = np.asarray(z, dtype=np.float64)[:V]
    if temperature <= 0.0:
        return int(np.argmax(z))
    x = z / temperature
    order = np.lexsort((np.arange(V), -x))          # x descending, index ascending
    keep = np.zeros(V, dtype=bool)
    k = V if (top_k <= 0 or top_k >= V) else top_k
    keep[order[:k]] = True
    w = np.where(keep, np.exp(x - np.max(x)), 0.0)
    if top_p < 1.0:
        total = w.sum()
        kept = order[:k]
        wk = w[kept]
        sub = np.lexsort((kept, -wk))                # weight descending, index ascending
        csum = np.cumsum(wk[sub])
        n = int(np.searchsorted(csum, top_p * total, side="left")) + 1
        keep2 = np.zeros(V, dtype=bool)
        keep2[kept[sub[:min(n, len(sub))]]] = True
        w = np.where(keep2, w, 0.0)
    c = np.cumsum(w)
    t = int(np.searchsorted(c, u * c[-1], side="right"))
    if t >= V:
        t = int(np.nonzero(w)[0][-1])
    return t


def sample_decode(cfg: OracleConfig, flat_params, prompt, n_new, temperature, top_k, top_p, uniforms,
                  dtype=np.float64):
    """Sampled continuation by full-prefix recomputation (no cache): each step
    draws the next token of every row with ``sample_token`` from the last
    position's logits and the row's uniform ``uniforms[b, step]``."""
    seq = np.asarray(prompt, dtype=np.int64)
    B = seq.shape[0]
    out = np.zeros((B, n_new), dtype=np.int64)
    for s in range(n_new):
        logits, _ = forward(cfg, flat_params, seq, None, dtype)
        last = logits.reshape(B, seq.shape[1], -1)[:, -1, :]
        for b in range(B):
            out[b, s] = sample_token(last[b], cfg.vocab, temperature, top_k, top_p, float(uniforms[b, s]))
        seq = np.concatenate([seq, out[:, s:s + 1]], axis=1)
    return out


# ---------------------------------------------------------------------------
# Beam search
# ---------------------------------------------------------------------------

def log_softmax_row(z, V):
    """log p over the real vocabulary 0..V-1 of one row of logits."""
    x = np.asarray(z[:V], dtype=np.float64)
    m = np.max(x)
    return x - (m + np.log(np.sum(np.exp(x - m))))


def beam_decode(cfg: OracleConfig, flat_params, prompt, n_new, width, dtype=np.float64):
    """Beam search by full-prefix recomputation (no cache).

    "RustGPT" lists beam search beside top-k / top-p and temperature among
    the sampling features its roadmap asks for (roadmap, "high-priority
    feature requests"); the page gives no further rule, so the plainest
    reading is taken: per prompt, keep the ``width`` continuations with the
    largest sum of next-token log-probabilities (log-softmax over the real
    vocabulary), extend every kept continuation by every token, keep the best
    ``width`` again, for exactly ``n_new`` tokens (no end token, no length
    normalisation).  Order: score descending, ties to the lower flat index
    parent_rank * V + token, where parent_rank is the parent's place in the
    previous step's order.  The first step extends the prompt alone.

    Returns (tokens [B, width, n_new], scores [B, width], margins [B, n_new]):
    beams best first; margins[b, s] is the gap between the last kept and the
    first dropped candidate at step s (inf where nothing was dropped).
    """
    prompt = np.asarray(prompt, dtype=np.int64)
    B, V = prompt.shape[0], cfg.vocab
    toks = np.zeros((B, width, n_new), dtype=np.int64)
    scores = np.zeros((B, width), dtype=np.float64)
    margins = np.zeros((B, n_new), dtype=np.float64)
    for b in range(B):
        beams = [(0.0, [])]                      # (score, tokens so far), best first
        for s in range(n_new):
            seqs = np.array([np.concatenate([prompt[b], np.array(t, dtype=np.int64)]) for _, t in beams])
            logits, _ = forward(cfg, flat_params, seqs, None, dtype)
            last = logits.reshape(len(beams), seqs.shape[1], -1)[:, -1, :]
            cand_score = np.concatenate([sc + log_softmax_row(last[r], V) for r, (sc, _) in enumerate(beams)])
            flat = np.arange(cand_score.size)
            order = np.lexsort((flat, -cand_score))   # score descending, then flat index ascending
            keep = order[:width]
            margins[b, s] = cand_score[keep[-1]] - cand_score[order[width]] if order.size > width else np.inf
            beams = [(float(cand_score[i]), beams[i // V][1] + [int(i % V)]) for i in keep]
        for w, (sc, t) in enumerate(beams):
            toks[b, w] = t
            scores[b, w] = sc
    return toks, scores, margins

