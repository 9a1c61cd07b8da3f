"""GPU parity of sampled decoding (temperature, top-k, top-p) against the oracle.

The random numbers are inputs (uniforms [B, n_new]), so both sides draw the
same tokens.  Check, per generated token: the oracle re-computes the logits of
the sequence the GPU generated (teacher-forced, full prefix, no cache) and
samples with the same uniform; the GPU's token must equal the oracle's, except
where the decision sits within a rounding margin of a boundary (the uniform
within 1e-4 of a cumulative-weight boundary), where it must equal the oracle's
choice for a uniform moved by that margin ("RustGPT", roadmap "high-priority
feature requests": temperature scaling, top-k, top-p).
"""
import numpy as np
import pytest

from oracle import gpt_oracle as O
from scratch_decoder_only_b200 import configs as CF
from tests.helpers import ocfg, tame_attention

pytestmark = pytest.mark.gpu

SETTINGS = [(1.0, 0, 1.0), (0.7, 20, 1.0), (1.3, 0, 0.8), (1.0, 40, 0.9), (2.0, 5, 0.5)]


@pytest.fixture(scope="module")
def torch():
    import torch as t
    assert t.cuda.is_available()
    return t


def dev(torch, a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def check_tokens(cfg, params, prompt, out, uni, temp, k, p, margin=1e-4):
    B, Tp = prompt.shape
    n_new = out.shape[1]
    seq = np.concatenate([prompt, out[:, :-1]], axis=1)
    z, _ = O.forward(cfg, params, seq)
    z = z.reshape(B, Tp + n_new - 1, -1)[:, Tp - 1:]
    near = 0
    for b in range(B):
        for s in range(n_new):
            u = float(uni[b, s])
            want = O.sample_token(z[b, s], cfg.vocab, temp, k, p, u)
            got = int(out[b, s])
            if got == want:
                continue
            # the inverse CDF runs in ascending token order, so the tokens that a
            # uniform within the margin can reach lie between these two
            lo_t, hi_t = (O.sample_token(z[b, s], cfg.vocab, temp, k, p, min(max(u + d, 0.0), 1 - 1e-12))
                          for d in (-margin, margin))
            assert lo_t <= got <= hi_t, (b, s, got, want, u, lo_t, hi_t)
            near += 1
    return near


@pytest.mark.parametrize("temp,k,p", SETTINGS)
def test_sample_decode_fp32_matches_oracle(torch, temp, k, p):
    from scratch_decoder_only_b200.gpt import GPT
    wl = CF.TINY_BYTE
    cfg = ocfg(wl.model)
    model = GPT(wl.model, 5)
    rng = np.random.default_rng(int(temp * 100) + k)
    B, Tp, n_new = 3, 10, 16
    prompt = rng.integers(0, 257, size=(B, Tp)).astype(np.int32)
    uni = rng.random((B, n_new)).astype(np.float32)
    out = model.sample_decode(dev(torch, prompt), n_new, dev(torch, uni), temp, k, p).cpu().numpy()
    assert model.status() == 0
    near = check_tokens(cfg, model.get_params().astype(np.float64), prompt, out, uni, temp, k, p)
    assert near <= 2
    if k:
        # every token lies in the oracle's top-k of its position
        assert out.min() >= 0 and out.max() < 257


def test_sample_decode_temperature_zero_is_greedy(torch):
    from scratch_decoder_only_b200.gpt import GPT
    wl = CF.TINY_BYTE
    model = GPT(wl.model, 6)
    rng = np.random.default_rng(3)
    prompt = dev(torch, rng.integers(0, 257, size=(2, 12)).astype(np.int32))
    uni = dev(torch, rng.random((2, 10)).astype(np.float32))
    a = model.sample_decode(prompt, 10, uni, 0.0, 0, 1.0).cpu().numpy()
    g = model.greedy_decode(prompt, 10).cpu().numpy()
    assert np.array_equal(a, g)
    # top_k = 1 is greedy for any temperature and uniform
    b = model.sample_decode(prompt, 10, uni, 1.7, 1, 1.0).cpu().numpy()
    assert np.array_equal(b, g)
    assert model.status() == 0


def test_sample_decode_inverse_cdf_over_rows(torch):
    """32 copies of one prompt with uniforms (b + 1/2) / 32: the first token of
    row b is the token whose cumulative-probability interval holds u_b, so the
    rows' first tokens follow the softmax at the prompt's last position."""
    from scratch_decoder_only_b200.gpt import GPT
    wl = CF.TINY_BYTE
    mc = CF.ModelConfig(**{**wl.model.as_dict(), "max_batch": 32})
    cfg = ocfg(mc)
    model = GPT(mc, 7)
    prompt = np.tile(np.arange(20, 32, dtype=np.int32), (32, 1))
    uni = ((np.arange(32) + 0.5) / 32).astype(np.float32)[:, None].repeat(2, axis=1)
    out = model.sample_decode(dev(torch, prompt), 2, dev(torch, uni), 1.0, 0, 1.0).cpu().numpy()
    z, _ = O.forward(cfg, model.get_params().astype(np.float64), prompt[:1])
    zl = z.reshape(12, -1)[-1, :mc.vocab]
    pr = np.exp(zl - zl.max())
    pr /= pr.sum()
    cdf = np.cumsum(pr)
    want = np.searchsorted(cdf, uni[:, 0], side="right")
    assert np.array_equal(out[:, 0], want)
    assert np.all(np.diff(out[:, 0]) >= 0)       # ascending u gives ascending tokens


def test_sample_decode_bf16_gpt2_shape(torch):
    """bf16 model with a 50304-column tied head (the GPT-2 vocabulary, the
    largest row the sampling kernel holds): temperature only, tokens checked
    against the oracle on the bf16-rounded weights with a uniform margin that
    covers bf16 activation rounding: logits off by up to about 0.1 shift the
    cumulative distribution by up to about that much (the exact sampling rule
    is pinned by the fp32 cases above)."""
    from scratch_decoder_only_b200.gpt import GPT
    mc = CF.ModelConfig(vocab=50257, vocab_padded=50304, d_model=128, n_heads=2, d_mlp=512, n_layers=2,
                        max_seq=64, max_batch=2, tied=True, precision="bf16", init_std=0.3)
    cfg = ocfg(mc)
    model = GPT(mc, 8)
    tame_attention(model, cfg)
    rng = np.random.default_rng(5)
    prompt = rng.integers(0, 50257, size=(2, 8)).astype(np.int32)
    uni = rng.random((2, 12)).astype(np.float32)
    out = model.sample_decode(dev(torch, prompt), 12, dev(torch, uni), 0.9, 0, 1.0).cpu().numpy()
    assert model.status() == 0
    p32 = model.get_params()
    u = p32.view(np.uint32)
    pb = ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).view(np.float32).astype(np.float64)
    near = check_tokens(cfg, pb, prompt, out, uni, 0.9, 0, 1.0, margin=0.1)
    assert near <= 8
