"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each test ties one part of the oracle to a closed form, an invariant, a
published known-answer value or finite differences, chosen so that a
plausible slip (a dropped term, a wrong sign or index, a transposed operand,
the wrong GELU or mask) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest

from oracle import gpt_oracle as O
from scratch_decoder_only_b200 import configs as CF
from scratch_decoder_only_b200 import synthetic as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def ocfg(mc: CF.ModelConfig) -> O.OracleConfig:
    return O.OracleConfig(vocab=mc.vocab, vocab_padded=mc.vocab_padded, d_model=mc.d_model,
                          n_heads=mc.n_heads, d_mlp=mc.d_mlp, n_layers=mc.n_layers,
                          max_seq=mc.max_seq, tied=mc.tied, ln_eps=mc.ln_eps,
                          init_std=mc.init_std, arch=mc.arch, n_kv_heads=mc.n_kv_heads, rope_base=mc.rope_base)


TINY = O.OracleConfig(vocab=11, vocab_padded=16, d_model=8, n_heads=2, d_mlp=16,
                      n_layers=2, max_seq=6)


def random_params(cfg, seed, scale=0.3):
    """Every parameter random (not the standard init), so each one matters."""
    rng = np.random.default_rng(seed)
    flat = rng.normal(0.0, scale, O.num_params(cfg))
    P = O.unflatten(cfg, flat)
    for name in P:
        if name.endswith("_g"):
            P[name][...] = 1.0 + rng.normal(0, 0.2, P[name].shape)
    P["wte"][cfg.vocab:] = 0.0
    if not cfg.tied:
        P["w_head"][cfg.vocab:] = 0.0
    return flat


# ---------------------------------------------------------------- generators

def test_splitmix64_known_answer():
    lines = [l for l in open(os.path.join(GOLDEN, "splitmix64_seed1234567.txt"))
             if l.strip() and not l.startswith("#")]
    seed = int(lines[0].split()[1])
    want = np.array([int(x) for x in lines[1:]], dtype=np.uint64)
    got = O.splitmix64(seed, np.arange(len(want), dtype=np.uint64))
    assert np.array_equal(got, want)


def test_box_muller_moments():
    z = O.gaussian_for_elements(7, np.arange(1_000_000, dtype=np.uint64))
    n = z.size
    assert abs(z.mean()) < 4 / math.sqrt(n)
    assert abs(z.std() - 1.0) < 4 * math.sqrt(0.5 / n)
    # fourth moment of N(0,1) is 3 (rules out uniform-like or mis-scaled draws)
    assert abs((z ** 4).mean() - 3.0) < 0.05
    # symmetric: the fraction below 0 is 1/2
    assert abs((z < 0).mean() - 0.5) < 4 * 0.5 / math.sqrt(n)


@pytest.mark.parametrize("wl,n_expected", [(CF.TINY_BYTE, 473_728), (CF.PACKED_SMALL, 4_950_144),
                                           (CF.BYTE_30M, 26_007_552), (CF.GPT2_124M, 124_475_904)])
def test_param_counts(wl, n_expected):
    assert O.num_params(ocfg(wl.model)) == n_expected
    assert wl.model.num_params() == n_expected


def test_init_statistics_and_constants():
    cfg = ocfg(CF.TINY_BYTE.model)
    flat = O.init_params(cfg, 42)
    P = O.unflatten(cfg, flat)
    for name, arr in P.items():
        leaf = name.split(".")[-1]
        if leaf.endswith("_g"):
            assert np.all(arr == 1.0)
        elif leaf.startswith("b_") or leaf.endswith("_b"):
            assert np.all(arr == 0.0)
        else:
            a = arr[:cfg.vocab] if leaf in ("wte", "w_head") else arr
            n = a.size
            assert abs(a.mean()) < 4 * 0.02 / math.sqrt(n), name
            assert abs(a.std() - 0.02) < 4 * 0.02 * math.sqrt(0.5 / n) + 1e-4, name
    # deterministic and seed-dependent
    assert np.array_equal(flat, O.init_params(cfg, 42))
    assert not np.array_equal(flat, O.init_params(cfg, 43))


def test_init_pad_rows_zero():
    cfg = O.OracleConfig(vocab=50, vocab_padded=64, d_model=16, n_heads=2, d_mlp=32,
                         n_layers=1, max_seq=8, tied=True)
    P = O.unflatten(cfg, O.init_params(cfg, 1))
    assert np.all(P["wte"][50:] == 0) and np.any(P["wte"][:50] != 0)


# ---------------------------------------------------------------- pieces

def test_positions_from_segments():
    pos, seg = O.positions_from_segments(np.array([[0, 0, 0, 1, 1, 2]]), 1, 6)
    assert pos.tolist() == [[0, 1, 2, 0, 1, 0]]
    pos, _ = O.positions_from_segments(None, 2, 4)
    assert pos.tolist() == [[0, 1, 2, 3]] * 2


def test_layernorm_hand_example():
    x = np.array([[1.0, 2.0, 3.0, 4.0]])
    y, xhat, rstd = O.layernorm_fwd(x, np.ones(4), np.zeros(4), 1e-5)
    # mean 2.5, biased variance 1.25
    want = (x - 2.5) / math.sqrt(1.25 + 1e-5)
    assert np.allclose(y, want, rtol=0, atol=1e-15)
    g, b = np.array([2.0, 1.0, 0.5, 3.0]), np.array([0.1, -0.2, 0.3, 0.0])
    y2, _, _ = O.layernorm_fwd(x, g, b, 1e-5)
    assert np.allclose(y2, want * g + b, atol=1e-15)
    rng = np.random.default_rng(0)
    z = rng.normal(3.0, 5.0, (7, 64))
    yz, _, _ = O.layernorm_fwd(z, np.ones(64), np.zeros(64), 0.0)
    assert np.allclose(yz.mean(-1), 0, atol=1e-12)
    assert np.allclose((yz ** 2).mean(-1), 1, atol=1e-12)


def test_gelu_tanh_form():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "gelu_tanh_points.txt"))
            if l.strip() and not l.startswith("#")]
    for u, g in rows:
        assert abs(O.gelu(np.float64(u)) - float(g)) < 1e-12
    assert abs(O.gelu(np.float64(1.0)) - 0.8413447460685429) > 1e-4   # not the erf form
    assert abs(O.gelu(np.float64(12.0)) - 12.0) < 1e-12
    assert abs(O.gelu(np.float64(-12.0))) < 1e-12
    u = np.linspace(-6, 6, 241)
    h = 1e-6
    fd = (O.gelu(u + h) - O.gelu(u - h)) / (2 * h)
    assert np.allclose(O.gelu_grad(u), fd, atol=1e-8)


def test_attention_hand_example():
    # one head, d = 4: scores scaled by 1/sqrt(4) = 1/2
    q = np.zeros((1, 1, 2, 4)); k = np.zeros((1, 1, 2, 4)); v = np.zeros((1, 1, 2, 4))
    q[0, 0, 1] = [2.0, 0, 0, 0]
    k[0, 0, 0] = [1.0, 0, 0, 0]
    v[0, 0, 0] = [1.0, 2.0, 3.0, 4.0]
    v[0, 0, 1] = [-1.0, 0.0, 1.0, 0.0]
    seg = np.zeros((1, 2), dtype=np.int64)
    o = O.attention_fwd(q, k, v, seg)
    # query 0 sees only key 0
    assert np.allclose(o[0, 0, 0], v[0, 0, 0], atol=0)
    # query 1: scores (1, 0) -> weights (e, 1)/(e+1)
    w0 = math.e / (math.e + 1)
    assert np.allclose(o[0, 0, 1], w0 * v[0, 0, 0] + (1 - w0) * v[0, 0, 1], atol=1e-15)
    # a new document at position 1: query 1 sees only itself
    o2 = O.attention_fwd(q, k, v, np.array([[0, 1]]))
    assert np.allclose(o2[0, 0, 1], v[0, 0, 1], atol=0)


def test_softmax_rows_sum_to_one():
    rng = np.random.default_rng(3)
    q, k = rng.normal(size=(3, 9, 8)), rng.normal(size=(3, 9, 8))
    seg = np.array([0, 0, 0, 1, 1, 1, 1, 2, 2])
    p = O.attention_probs(q, k, O.allowed_mask(seg))
    assert np.all(np.abs(p.sum(-1) - 1.0) <= 1e-12)
    assert np.all(p[:, ~O.allowed_mask(seg)] == 0.0)
    p32 = O.attention_probs(q.astype(np.float32), k.astype(np.float32), O.allowed_mask(seg))
    assert np.all(np.abs(p32.sum(-1) - 1.0) <= 1e-6)
    z = rng.normal(size=(5, 20))
    _, dz = O.cross_entropy(z, np.array([1, 2, 3, 4, 5]), 20)
    assert np.allclose(dz.sum(1), 0.0, atol=1e-15)   # softmax rows sum to 1 minus the one-hot


def test_cross_entropy_closed_forms():
    V = 7
    z = np.zeros((3, 10))
    loss, dz = O.cross_entropy(z, np.array([0, 6, -1]), V)
    assert abs(loss - math.log(V)) < 1e-15
    assert np.all(dz[:, V:] == 0) and np.all(dz[2] == 0)
    assert abs(dz[0, 0] - (1 / V - 1) / 2) < 1e-15 and abs(dz[0, 1] - (1 / V) / 2) < 1e-15
    # hand example, V = 3, logits (0, ln 2, 0), target 1: p = (1/4, 1/2, 1/4), loss = ln 2
    z = np.array([[0.0, math.log(2.0), 0.0]])
    loss, dz = O.cross_entropy(z, np.array([1]), 3)
    assert abs(loss - math.log(2.0)) < 1e-15
    assert np.allclose(dz, [[0.25, -0.5, 0.25]], atol=1e-15)


# ---------------------------------------------------------------- whole model

def _fd_check(cfg, seg, seed):
    rng = np.random.default_rng(seed)
    B, T = 2, cfg.max_seq
    x = rng.integers(0, cfg.vocab, size=(B, T + 1))
    tokens, targets = x[:, :-1], x[:, 1:].copy()
    if seg is not None:
        targets[:, :-1][seg[:, 1:] != seg[:, :-1]] = -1
    targets[0, 2] = -1                       # an ignored position
    flat = random_params(cfg, seed)
    loss, g = O.loss_and_grads(cfg, flat, tokens, targets, seg)
    h = 1e-5
    fd = np.empty_like(g)
    for i in range(flat.size):
        old = flat[i]
        flat[i] = old + h
        lp, _ = O.cross_entropy(O.forward(cfg, flat, tokens, seg)[0], targets.reshape(-1), cfg.vocab)
        flat[i] = old - h
        lm, _ = O.cross_entropy(O.forward(cfg, flat, tokens, seg)[0], targets.reshape(-1), cfg.vocab)
        flat[i] = old
        fd[i] = (lp - lm) / (2 * h)
    err = np.abs(fd - g) - 1e-6 * np.maximum(1.0, np.abs(g))
    assert np.all(err <= 0), (np.max(np.abs(fd - g)), int(np.argmax(err)))
    # the check must see real gradients in every tensor class
    assert np.count_nonzero(g) > 0.5 * g.size
    return g


def test_fd_gradients_plain():
    _fd_check(TINY, None, 11)


def test_fd_gradients_packed():
    seg = np.array([[0, 0, 0, 1, 1, 1], [0, 0, 1, 1, 1, 2]])
    _fd_check(TINY, seg, 12)


def test_fd_gradients_tied():
    cfg = O.OracleConfig(**{**TINY.__dict__, "tied": True})
    _fd_check(cfg, None, 13)


def test_block_structure_with_zero_input_weights():
    """With every block's input projections zero (W_qkv = W_fc = 0) each block
    adds a position-independent vector to the residual stream, computable by
    hand: attention rows are convex combinations of identical value rows, so
    each head returns its slice of the value bias b_qkv[2C:3C]; the MLP sees
    u = b_fc.  Hence x_L = wte[tok] + wpe[pos] + sum over blocks of
    (b_v W_o^T + b_o + gelu(b_fc) W_fc2^T + b_fc2) and the logits are
    LN_f(x_L) W_head^T.  Pins the pre-LN residual wiring, the [out, in]
    weight orientation, the q/k/v order inside W_qkv and b_qkv, the final
    LayerNorm and the head, none of which finite differences can see."""
    cfg = O.OracleConfig(vocab=13, vocab_padded=16, d_model=8, n_heads=2, d_mlp=12, n_layers=3, max_seq=7)
    flat = random_params(cfg, 31)
    P = O.unflatten(cfg, flat)                     # views into flat
    C = cfg.d_model
    for l in range(cfg.n_layers):
        P[f"h{l}.w_qkv"][...] = 0.0
        P[f"h{l}.w_fc"][...] = 0.0
    rng = np.random.default_rng(32)
    tok = rng.integers(0, cfg.vocab, size=(2, 7))
    logits, _ = O.forward(cfg, flat, tok)

    def gelu_tanh(u):
        return 0.5 * u * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (u + 0.044715 * u ** 3)))

    x = P["wte"][tok] + P["wpe"][np.arange(7)][None, :, :]
    for l in range(cfg.n_layers):
        b_v = P[f"h{l}.b_qkv"][2 * C:3 * C]
        x = x + b_v @ P[f"h{l}.w_o"].T + P[f"h{l}.b_o"]
        x = x + gelu_tanh(P[f"h{l}.b_fc"]) @ P[f"h{l}.w_fc2"].T + P[f"h{l}.b_fc2"]
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    xf = (x - mu) / np.sqrt(var + cfg.ln_eps) * P["lnf_g"] + P["lnf_b"]
    want = xf.reshape(-1, C) @ P["w_head"].T
    assert np.allclose(logits, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("tied", [False, True])
def test_padded_vocab_columns_take_no_part(tied):
    """Columns V..Vp-1 of the LM head are padding: the loss, the gradient of
    every real parameter and greedy decoding ignore whatever sits in the pad
    rows, and the pad rows' own gradient is exactly zero."""
    cfg = O.OracleConfig(**{**TINY.__dict__, "tied": tied})
    flat = random_params(cfg, 21)
    rng = np.random.default_rng(22)
    tok = rng.integers(0, cfg.vocab, size=(2, 6))
    tgt = rng.integers(0, cfg.vocab, size=(2, 6))
    loss0, g0 = O.loss_and_grads(cfg, flat, tok, tgt)
    head = "wte" if tied else "w_head"
    flat_big = flat.copy()
    big = O.unflatten(cfg, flat_big)              # views into flat_big
    big[head][cfg.vocab:] = rng.normal(0.0, 50.0, big[head][cfg.vocab:].shape)   # huge pad logits
    loss1, g1 = O.loss_and_grads(cfg, flat_big, tok, tgt)
    assert loss1 == loss0
    G0, G1 = O.unflatten(cfg, g0), O.unflatten(cfg, g1)
    for k in G0:
        if tied and k == "w_head":               # an alias of wte
            continue
        if k == head:
            assert np.array_equal(G1[k][:cfg.vocab], G0[k][:cfg.vocab])
            assert not np.any(G1[k][cfg.vocab:]) and not np.any(G0[k][cfg.vocab:])
        else:
            assert np.array_equal(G1[k], G0[k]), k
    d0, _ = O.greedy_decode(cfg, flat, tok[:, :3], 3, dtype=np.float64)
    d1, _ = O.greedy_decode(cfg, flat_big, tok[:, :3], 3, dtype=np.float64)
    assert np.array_equal(d0, d1) and d1.max() < cfg.vocab


def test_initial_loss_near_ln_v():
    wl = CF.TINY_BYTE
    cfg = ocfg(wl.model)
    flat = O.init_params(cfg, wl.init_seed)
    tok, tgt, seg = S.make_batch(wl)
    logits, _ = O.forward(cfg, flat, tok, seg)
    loss, _ = O.cross_entropy(logits, tgt.reshape(-1), cfg.vocab)
    sigma2 = cfg.init_std ** 2 * cfg.d_model
    assert abs(loss - (math.log(cfg.vocab) + sigma2 / 2)) <= 0.1
    assert abs(math.log(257) - 5.5491) < 1e-4


def test_mask_future_has_no_influence():
    cfg = TINY
    flat = random_params(cfg, 5)
    rng = np.random.default_rng(5)
    tok = rng.integers(0, cfg.vocab, size=(2, 6))
    for seg in (None, np.array([[0, 0, 0, 1, 1, 1], [0, 1, 1, 1, 2, 2]])):
        base, _ = O.forward(cfg, flat, tok, seg)
        base = base.reshape(2, 6, -1)
        for j in range(6):
            t2 = tok.copy()
            t2[:, j] = (t2[:, j] + 1) % cfg.vocab
            alt = O.forward(cfg, flat, t2, seg)[0].reshape(2, 6, -1)
            for b in range(2):
                for i in range(6):
                    same_doc = seg is None or seg[b, i] == seg[b, j]
                    if i < j or not same_doc:
                        assert np.array_equal(base[b, i], alt[b, i]), (b, i, j)
                    elif i == j:
                        assert not np.array_equal(base[b, i], alt[b, i])


def test_packed_row_equals_separate_documents():
    cfg = TINY
    flat = random_params(cfg, 8)
    rng = np.random.default_rng(8)
    tok = rng.integers(0, cfg.vocab, size=(1, 6))
    seg = np.array([[0, 0, 0, 0, 1, 1]])
    packed, _ = O.forward(cfg, flat, tok, seg)
    a, _ = O.forward(cfg, flat, tok[:, :4], None)
    b, _ = O.forward(cfg, flat, tok[:, 4:], None)
    assert np.allclose(packed[:4], a, rtol=0, atol=1e-12)
    assert np.allclose(packed[4:], b, rtol=0, atol=1e-12)
    # all-equal seg ids is plain causal
    same, _ = O.forward(cfg, flat, tok, np.zeros((1, 6), dtype=np.int64))
    plain, _ = O.forward(cfg, flat, tok, None)
    assert np.array_equal(same, plain)


# ---------------------------------------------------------------- optimiser

def test_clip_coefficient_hand_vector():
    norm, coef = O.clip_coefficient(np.array([3.0, 4.0]), 1.0)
    assert norm == 5.0 and abs(coef - 1.0 / (5.0 + 1e-6)) < 1e-18
    norm, coef = O.clip_coefficient(np.array([0.3, 0.4]), 1.0)
    assert coef == 1.0


def test_adamw_closed_forms():
    lr, b1, b2, eps, wd = 1e-3, 0.9, 0.95, 1e-8, 0.1
    p0 = np.array([0.5, -0.25, 0.0, 1.0])
    g1 = np.array([0.2, -0.1, 0.0, 3.0])
    p1, m1, v1 = O.adamw_update(p0, g1, np.zeros(4), np.zeros(4), 1, lr, b1, b2, eps, wd)
    # step 1: m_hat = g, v_hat = g^2 -> update = g/(|g|+eps)
    want1 = p0 - lr * (g1 / (np.abs(g1) + eps) + wd * p0)
    assert np.allclose(p1, want1, rtol=0, atol=1e-15)
    # step 2 by hand in plain Python floats for element 0
    g2 = 0.05
    m = b1 * (1 - b1) * 0.2 + (1 - b1) * g2
    v = b2 * (1 - b2) * 0.04 + (1 - b2) * g2 * g2
    mh, vh = m / (1 - b1 ** 2), v / (1 - b2 ** 2)
    want = p1[0] - lr * (mh / (math.sqrt(vh) + eps) + wd * p1[0])
    p2, _, _ = O.adamw_update(p1, np.array([g2, 0, 0, 0]), m1, v1, 2, lr, b1, b2, eps, wd)
    assert abs(p2[0] - want) < 1e-16


def test_clip_adamw_step_skips_nonfinite():
    p = np.ones(3); g = np.array([1.0, np.inf, 0.0])
    p2, m2, v2, norm, skipped = O.clip_adamw_step(p, g, np.zeros(3), np.zeros(3), 1,
                                                  1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0)
    assert skipped and np.array_equal(p2, p)
    # clipped step: clip coefficient cancels at t = 1 except through eps
    g = np.array([30.0, 40.0, 0.0])
    p2, _, _, norm, skipped = O.clip_adamw_step(p, g, np.zeros(3), np.zeros(3), 1,
                                                1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0)
    assert not skipped and norm == 50.0
    assert np.allclose(p2, [1 - 1e-3, 1 - 1e-3, 1.0], atol=1e-9)


def test_loss_scale_rule():
    s, good, skip = O.loss_scale_update(2.0 ** 15, 5, False)
    assert (s, good, skip) == (2.0 ** 14, 0, True)
    s, good = 2.0 ** 15, 0
    for _ in range(1999):
        s, good, skip = O.loss_scale_update(s, good, True)
    assert s == 2.0 ** 15 and good == 1999
    s, good, skip = O.loss_scale_update(s, good, True)
    assert s == 2.0 ** 16 and good == 0 and not skip


# ---------------------------------------------------------------- decoding

def _successor_model(V, C):
    """Blocks are identities (zero weights), positions are 0, token k embeds as
    the k-th unit vector and the head row c reads coordinate (c-1) mod V, so the
    next token after k is (k+1) mod V."""
    cfg = O.OracleConfig(vocab=V, vocab_padded=V, d_model=C, n_heads=2, d_mlp=2 * C,
                         n_layers=2, max_seq=16)
    flat = np.zeros(O.num_params(cfg))
    P = O.unflatten(cfg, flat)
    for name in P:
        if name.endswith("_g"):
            P[name][...] = 1.0
    P["wte"][np.arange(V), np.arange(V)] = 1.0
    P["w_head"][np.arange(V), (np.arange(V) - 1) % V] = 1.0
    return cfg, flat


def test_greedy_decode_successor_model():
    cfg, flat = _successor_model(V=6, C=8)
    out, gaps = O.greedy_decode(cfg, flat, np.array([[0, 3], [2, 5]]), n_new=5, dtype=np.float64)
    assert out.tolist() == [[4, 5, 0, 1, 2], [0, 1, 2, 3, 4]]
    assert np.all(gaps > 0)


def test_greedy_decode_tie_lowest_index():
    cfg, flat = _successor_model(V=6, C=8)
    P = O.unflatten(cfg, flat)
    P["w_head"][2] = P["w_head"][5]          # column 2 ties with column 5
    out, gaps = O.greedy_decode(cfg, flat, np.array([[4]]), n_new=1, dtype=np.float64)
    assert out.tolist() == [[2]] and gaps[0, 0] == 0.0


def test_lr_schedule_special_points():
    """Cosine schedule with warm-up ("LucilleAI", "Getting started": cosine,
    warm-up steps, min-lr): checked at points fixed by the shape alone, not by
    retyping the formula -- the ramp's first value and its top, the decay's
    start at max_lr, its end at min_lr, the midpoint at the mean of the two,
    the mirror symmetry lr(r) + lr(1 - r) = max + min of half a cosine period,
    monotone decay, and the constant kind."""
    kw = dict(kind=1, warmup=100, total=1100, max_lr=6e-4, min_lr=3e-5)
    assert O.lr_at(0, **kw) == pytest.approx(6e-6, rel=1e-12)
    assert O.lr_at(99, **kw) == pytest.approx(6e-4, rel=1e-12)
    assert O.lr_at(100, **kw) == pytest.approx(6e-4, rel=1e-12)
    assert O.lr_at(600, **kw) == pytest.approx((6e-4 + 3e-5) / 2, rel=1e-12)
    assert O.lr_at(1100, **kw) == pytest.approx(3e-5, rel=1e-12)
    assert O.lr_at(5000, **kw) == pytest.approx(3e-5, rel=1e-12)
    for d in (1, 37, 250, 499):
        assert O.lr_at(100 + d, **kw) + O.lr_at(1100 - d, **kw) == pytest.approx(6e-4 + 3e-5, rel=1e-12)
    seq = [O.lr_at(s, **kw) for s in range(100, 1101)]
    assert all(a >= b for a, b in zip(seq, seq[1:]))
    # the ramp is linear: equal increments
    ramp = np.diff([O.lr_at(s, **kw) for s in range(100)])
    assert np.allclose(ramp, 6e-6, rtol=1e-9)
    assert O.lr_at(12, kind=0, warmup=0, total=1, max_lr=1.0, min_lr=0.0, lr_const=2.5e-4) == 2.5e-4


def test_sampling_reduces_to_greedy_and_inverse_cdf():
    """Sampling ("RustGPT" roadmap: temperature scaling, top-k, top-p):
    pinned by the cases that reduce to something known -- temperature 0 and
    top-k = 1 are greedy (lowest index on ties); with no top-k / top-p, a grid
    of N uniforms (i + 1/2)/N lands on each token about N * softmax(z / T)
    times (the inverse-CDF property), at T = 1 and T = 2; top-k keeps exactly
    the k largest logits with ties to the lower index; top-p on a hand example
    keeps the smallest high-probability prefix."""
    rng = np.random.default_rng(12)
    z = rng.normal(0, 2.0, 50)
    V = 50
    assert O.sample_token(z, V, 0.0, 0, 1.0, 0.7) == int(np.argmax(z))
    for u in (0.0, 0.3, 0.999):
        assert O.sample_token(z, V, 1.3, 1, 1.0, u) == int(np.argmax(z))
    zt = np.array([1.0, 2.0, 2.0, 0.0])
    assert O.sample_token(zt, 4, 1.0, 1, 1.0, 0.9) == 1
    assert {O.sample_token(zt, 4, 1.0, 2, 1.0, u) for u in np.linspace(0, 0.999, 200)} == {1, 2}
    N = 20000
    for T in (1.0, 2.0):
        p = np.exp(z / T - np.max(z / T))
        p /= p.sum()
        counts = np.bincount([O.sample_token(z, V, T, 0, 1.0, (i + 0.5) / N) for i in range(N)], minlength=V)
        assert np.all(np.abs(counts - N * p) <= 1.0 + 1e-9), np.max(np.abs(counts - N * p))
    # top-k = 5 at T = 1: only the five largest appear, in proportion to their renormalised softmax
    top5 = np.argsort(-z)[:5]
    p5 = np.exp(z[top5] - z[top5].max())
    p5 /= p5.sum()
    counts = np.bincount([O.sample_token(z, V, 1.0, 5, 1.0, (i + 0.5) / N) for i in range(N)], minlength=V)
    assert set(np.nonzero(counts)[0]) == set(top5)
    assert np.all(np.abs(counts[top5] - N * p5) <= 1.0 + 1e-9)
    # top-p: probabilities (0.5, 0.3, 0.15, 0.05)
    zp = np.log([0.15, 0.5, 0.05, 0.3])
    assert {O.sample_token(zp, 4, 1.0, 0, 0.6, u) for u in np.linspace(0, 0.999, 100)} == {1, 3}
    assert {O.sample_token(zp, 4, 1.0, 0, 0.85, u) for u in np.linspace(0, 0.999, 100)} == {0, 1, 3}
    assert {O.sample_token(zp, 4, 1.0, 0, 0.4, u) for u in np.linspace(0, 0.999, 100)} == {1}
    # in ascending token order: with (1, 3) kept, u below 0.5 / 0.8 gives token 1
    assert O.sample_token(zp, 4, 1.0, 0, 0.6, 0.6) == 1 and O.sample_token(zp, 4, 1.0, 0, 0.6, 0.65) == 3


# ---------------------------------------------------------------- Llama-style block

LLAMA = O.OracleConfig(vocab=11, vocab_padded=16, d_model=16, n_heads=4, d_mlp=12, n_layers=2, max_seq=6,
                       arch="llama", n_kv_heads=2)


@pytest.mark.parametrize("variant", ["plain", "packed", "tied", "mha"])
def test_llama_fd_gradients(variant):
    """Central finite differences on every parameter element of the Llama-style
    block (RMSNorm, rotary positions, two query heads per key / value head,
    SwiGLU); packed rows restart the rotary positions at each document."""
    cfg = LLAMA
    seg = None
    if variant == "packed":
        seg = np.array([[0, 0, 0, 1, 1, 1], [0, 0, 1, 1, 1, 2]])
    elif variant == "tied":
        cfg = O.OracleConfig(**{**LLAMA.__dict__, "tied": True})
    elif variant == "mha":
        cfg = O.OracleConfig(**{**LLAMA.__dict__, "n_kv_heads": 4})
    _fd_check(cfg, seg, 21)


def test_rope_scores_depend_on_relative_position_only():
    """Rotary positions (Su et al., RoFormer): a rotated query at position i
    against a rotated key at position j gives the same score for every shift
    (i + s, j + s), and the rotation keeps the vector norm; the inverse
    rotation undoes it."""
    rng = np.random.default_rng(5)
    d = 16
    q = rng.normal(size=(1, 1, 1, d))
    k = rng.normal(size=(1, 1, 1, d))

    def rot(x, p):
        return O.rope_apply(x, O.rope_angles(np.array([[p]]), d, 10000.0))

    base = float((rot(q, 7) * rot(k, 3)).sum())
    for s in (1, 5, 100, 1000):
        assert float((rot(q, 7 + s) * rot(k, 3 + s)).sum()) == pytest.approx(base, rel=1e-9, abs=1e-9)
    assert float((rot(q, 7) * rot(k, 4)).sum()) != pytest.approx(base, rel=1e-6)
    assert np.linalg.norm(rot(q, 123)) == pytest.approx(np.linalg.norm(q), rel=1e-12)
    ang = O.rope_angles(np.array([[9]]), d, 10000.0)
    assert np.allclose(O.rope_apply(O.rope_apply(q, ang), ang, inverse=True), q, atol=1e-12)
    # position 0 is the identity
    assert np.array_equal(rot(q, 0), q)


def test_gqa_equals_mha_with_repeated_key_value_heads():
    """Two query heads per key / value head give exactly the logits of the
    multi-head model whose key and value weights repeat each shared head."""
    cfg = LLAMA
    mha = O.OracleConfig(**{**LLAMA.__dict__, "n_kv_heads": 4})
    flat = random_params(cfg, 41)
    P = O.unflatten(cfg, flat)
    Q = O.unflatten(mha, np.zeros(O.num_params(mha)))
    C, d, Hkv, G = cfg.d_model, cfg.head_dim, cfg.kv_heads, cfg.n_heads // cfg.kv_heads
    for name in P:
        if name.endswith("w_qkv"):
            w = P[name]
            q_rows = w[:C]
            k_rows = w[C:C + Hkv * d].reshape(Hkv, d, C)
            v_rows = w[C + Hkv * d:].reshape(Hkv, d, C)
            Q[name][...] = np.concatenate([q_rows, np.repeat(k_rows, G, axis=0).reshape(-1, C),
                                           np.repeat(v_rows, G, axis=0).reshape(-1, C)])
        else:
            Q[name][...] = P[name]
    tok = np.random.default_rng(42).integers(0, cfg.vocab, size=(2, 6))
    qflat = np.concatenate([Q[n].reshape(-1) for n, _ in O.param_shapes(mha)])
    a, _ = O.forward(cfg, flat, tok)
    b, _ = O.forward(mha, qflat, tok)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-12)


def test_rmsnorm_and_silu_special_cases():
    """RMSNorm of a constant row c is sign(c) |c| / sqrt(c^2 + eps) times the
    gain, and scaling a row leaves RMSNorm unchanged when eps = 0; silu(0) = 0,
    silu(z) -> z for large z and -> 0 for very negative z; silu' matches a
    central difference."""
    g = np.arange(1, 9, dtype=np.float64)
    y, _, _ = O.rmsnorm_fwd(np.full((1, 8), -3.0), g, 1e-5)
    assert np.allclose(y, -3.0 / math.sqrt(9.0 + 1e-5) * g)
    x = np.random.default_rng(3).normal(size=(2, 8))
    assert np.allclose(O.rmsnorm_fwd(x, g, 0.0)[0], O.rmsnorm_fwd(7.5 * x, g, 0.0)[0])
    assert O.silu(np.array(0.0)) == 0.0
    assert O.silu(np.array(40.0)) == pytest.approx(40.0, rel=1e-12)
    assert abs(O.silu(np.array(-40.0))) < 1e-15
    z = np.linspace(-6, 6, 25)
    fd = (O.silu(z + 1e-6) - O.silu(z - 1e-6)) / 2e-6
    assert np.allclose(O.silu_grad(z), fd, atol=1e-8)


def test_llama_mask_and_packing_bit_identity():
    """Changing token j leaves the logits of earlier positions bit-identical,
    and a packed row equals its documents run separately (positions restart)."""
    cfg = LLAMA
    flat = random_params(cfg, 43)
    rng = np.random.default_rng(44)
    tok = rng.integers(0, cfg.vocab, size=(1, 6))
    a, _ = O.forward(cfg, flat, tok)
    t2 = tok.copy()
    t2[0, 4] = (t2[0, 4] + 1) % cfg.vocab
    b, _ = O.forward(cfg, flat, t2)
    assert np.array_equal(a[:4], b[:4]) and not np.array_equal(a[4], b[4])
    seg = np.array([[0, 0, 0, 1, 1, 1]])
    p, _ = O.forward(cfg, flat, tok, seg)
    d0, _ = O.forward(cfg, flat, tok[:, :3])
    d1, _ = O.forward(cfg, flat, tok[:, 3:])
    assert np.array_equal(p[:3], d0) and np.array_equal(p[3:], d1)


# ---------------------------------------------------------------------------
# Beam search
# ---------------------------------------------------------------------------

def _seq_logprob_bruteforce(cfg, flat, prompt_row, cont):
    """Total log-probability of a continuation from ONE forward pass over the
    whole sequence (not step by step), log-softmax by scipy's logsumexp over
    the real vocabulary."""
    from scipy.special import logsumexp
    seq = np.concatenate([prompt_row, cont])[None, :]
    z, _ = O.forward(cfg, flat, seq, None, np.float64)
    z = z.reshape(seq.shape[1], -1)[:, :cfg.vocab]
    Tp = prompt_row.size
    tot = 0.0
    for i, t in enumerate(cont):
        row = z[Tp - 1 + i]
        tot += row[t] - logsumexp(row)
    return tot


def test_beam_exhaustive_when_width_covers_all_prefixes():
    """With V = 3 and width 9 = V^2, the last step ranks every one of the 27
    three-token continuations, so the beams are exactly the 9 best sequences
    by total log-probability (each scored here by one full-sequence forward)."""
    import itertools
    cfg = O.OracleConfig(vocab=3, vocab_padded=8, d_model=8, n_heads=2, d_mlp=16, n_layers=2, max_seq=8)
    flat = random_params(cfg, 61, scale=0.8)
    prompt = np.array([[1, 0, 2], [2, 2, 1]])
    toks, scores, _ = O.beam_decode(cfg, flat, prompt, 3, 9)
    for b in range(2):
        allseq = [np.array(c) for c in itertools.product(range(3), repeat=3)]
        lp = np.array([_seq_logprob_bruteforce(cfg, flat, prompt[b], c) for c in allseq])
        order = np.argsort(-lp, kind="stable")[:9]
        assert np.allclose(scores[b], lp[order], rtol=0, atol=1e-12)
        for w in range(9):
            assert np.array_equal(toks[b, w], allseq[order[w]])


def test_beam_width_one_is_greedy_and_scores_are_log_probs():
    """Width 1 keeps the argmax every step (greedy decoding); every beam's
    score is its continuation's total log-probability; scores descend; the
    beams are distinct."""
    cfg = O.OracleConfig(vocab=50, vocab_padded=64, d_model=16, n_heads=2, d_mlp=32, n_layers=2, max_seq=12)
    flat = random_params(cfg, 62, scale=0.5)
    prompt = np.array([[3, 7, 11, 2], [9, 9, 40, 1]])
    g, _ = O.greedy_decode(cfg, flat, prompt, 5, dtype=np.float64)
    t1, _, _ = O.beam_decode(cfg, flat, prompt, 5, 1)
    assert np.array_equal(t1[:, 0], g)
    toks, scores, margins = O.beam_decode(cfg, flat, prompt, 5, 4)
    for b in range(2):
        assert np.all(np.diff(scores[b]) <= 0)
        assert len({tuple(t) for t in toks[b]}) == 4
        for w in range(4):
            assert abs(scores[b, w] - _seq_logprob_bruteforce(cfg, flat, prompt[b], toks[b, w])) < 1e-10
    # a wider beam never ends below the narrower one's best
    assert np.all(scores[:, 0] >= O.beam_decode(cfg, flat, prompt, 5, 2)[1][:, 0] - 1e-12)
    assert np.all(margins >= 0)


def test_beam_ties_go_to_lower_flat_index():
    """A model whose logits ignore the input (zero weights, zero head): every
    token has log-probability -log V, so the beams after two steps are the
    lexicographically first continuations (0,0), (0,1), ..."""
    cfg = O.OracleConfig(vocab=5, vocab_padded=8, d_model=8, n_heads=2, d_mlp=16, n_layers=1, max_seq=6)
    flat = np.zeros(O.num_params(cfg))
    toks, scores, margins = O.beam_decode(cfg, flat, np.array([[1, 2]]), 2, 3)
    assert np.array_equal(toks[0], [[0, 0], [0, 1], [0, 2]])
    assert np.allclose(scores, -2 * np.log(5))
    assert np.all(margins == 0)
