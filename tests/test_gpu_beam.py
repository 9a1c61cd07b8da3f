"""Beam search on the GPU against the oracle's beam search ("RustGPT",
roadmap "high-priority feature requests": beam search).

* fp32, head size 64: beams, their order and their scores equal the oracle's
  (fp64) wherever every step's margin between the last kept and the first
  dropped candidate exceeds 1e-4 (fp32 logits differ from fp64 by ~1e-6);
* width 1 is greedy decoding;
* bf16, batch x width = 8 (GEMV projections) and 12 (tensor-core GEMM), and
  the Llama-style block (grouped key/value heads read through the source-row
  table): every beam's score equals the oracle's log-probability of its
  tokens (one full-sequence forward on the bf16-rounded weights) within the
  16-bit tolerance, beams distinct and ordered;
* argument checks.
"""
import numpy as np
import pytest

from oracle import gpt_oracle as O
from scratch_decoder_only_b200 import configs as CF
from scratch_decoder_only_b200 import synthetic as S
from tests.helpers import ocfg, tame_attention

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch as t
    assert t.cuda.is_available()
    return t


def dev(torch, a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bf16_round(p32):
    u = p32.astype(np.float32).view(np.uint32)
    r = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return r.view(np.float32).astype(np.float64)


def seq_logprob(cfg, params, prompt_row, cont):
    """log-probability of a continuation from one full-sequence forward."""
    seq = np.concatenate([prompt_row, cont])[None, :]
    z, _ = O.forward(cfg, params, seq)
    z = z.reshape(seq.shape[1], -1)[:, :cfg.vocab]
    Tp = prompt_row.size
    tot, per = 0.0, []
    for i, t in enumerate(cont):
        row = z[Tp - 1 + i]
        m = row.max()
        lp = row[t] - (m + np.log(np.exp(row - m).sum()))
        tot += lp
        per.append(np.abs(row).max())
    return tot, np.array(per)


FP32_64 = CF.ModelConfig(vocab=2000, vocab_padded=2000, d_model=256, n_heads=4, d_mlp=512, n_layers=2,
                         max_seq=48, max_batch=8, tied=True, precision="fp32", init_std=0.5)


@pytest.mark.parametrize("seed", [6, 8])
def test_beam_fp32_matches_oracle(torch, seed):
    from scratch_decoder_only_b200.gpt import GPT
    cfg = ocfg(FP32_64)
    model = GPT(FP32_64, 17)
    prompt = S.make_prompts(CF.GPT2_DECODE, 2, prompt_len=12, seed=seed) % FP32_64.vocab
    toks, scores = model.beam_decode(dev(torch, prompt.astype(np.int32)), 12, 4)
    toks, scores = toks.cpu().numpy(), scores.cpu().numpy()
    assert model.status() == 0
    ref_t, ref_s, margins = O.beam_decode(cfg, model.get_params().astype(np.float64), prompt, 12, 4)
    assert margins.min() > 1e-4, margins.min()
    assert np.array_equal(toks, ref_t), (toks, ref_t)
    assert np.max(np.abs(scores - ref_s)) <= 1e-4, np.max(np.abs(scores - ref_s))


def test_beam_width_one_is_greedy(torch):
    from scratch_decoder_only_b200.gpt import GPT
    cfg = ocfg(FP32_64)
    model = GPT(FP32_64, 17)
    prompt = (S.make_prompts(CF.GPT2_DECODE, 3, prompt_len=10, seed=11) % FP32_64.vocab).astype(np.int32)
    g = model.greedy_decode(dev(torch, prompt), 15).cpu().numpy()
    t1, s1 = model.beam_decode(dev(torch, prompt), 15, 1)
    assert model.status() == 0
    assert np.array_equal(t1.cpu().numpy()[:, 0], g)
    _, gaps = O.greedy_decode(cfg, model.get_params(), prompt, 15, dtype=np.float32)
    assert gaps.min() > 1e-5


def check_beams(cfg, params, prompt, toks, scores, W, rel_tol=0.01):
    """Scores ordered, beams distinct, each score the oracle's log-probability
    of the beam's tokens within rel_tol of the logit scale per token."""
    for b in range(prompt.shape[0]):
        assert np.all(np.diff(scores[b]) <= 0), scores[b]
        assert len({tuple(t) for t in toks[b]}) == W
        for w in range(W):
            lp, scale = seq_logprob(cfg, params, prompt[b], toks[b, w])
            tol = 2 * rel_tol * scale.sum()
            assert abs(scores[b, w] - lp) <= tol, (b, w, scores[b, w], lp, tol)


DEC64 = CF.ModelConfig(vocab=1000, vocab_padded=1024, d_model=256, n_heads=4, d_mlp=1024, n_layers=2,
                       max_seq=64, max_batch=12, tied=False, precision="bf16", init_std=0.3)


@pytest.mark.parametrize("B", [2, 3])
def test_beam_bf16_scores_are_log_probs(torch, B):
    from scratch_decoder_only_b200.gpt import GPT
    cfg = ocfg(DEC64)
    model = GPT(DEC64, 13)
    tame_attention(model, cfg)
    rng = np.random.default_rng(70 + B)
    prompt = rng.integers(0, DEC64.vocab, size=(B, 16)).astype(np.int32)
    toks, scores = model.beam_decode(dev(torch, prompt), 20, 4)
    assert model.status() == 0
    check_beams(cfg, bf16_round(model.get_params()), prompt, toks.cpu().numpy(), scores.cpu().numpy(), 4)


def test_beam_llama_bf16(torch):
    from scratch_decoder_only_b200.gpt import GPT
    mc = CF.ModelConfig(vocab=1000, vocab_padded=1024, d_model=256, n_heads=4, d_mlp=672, n_layers=2,
                        max_seq=64, max_batch=12, tied=False, precision="bf16", arch="llama", n_kv_heads=2,
                        init_std=0.3)
    cfg = ocfg(mc)
    model = GPT(mc, 14)
    tame_attention(model, cfg)
    rng = np.random.default_rng(77)
    prompt = rng.integers(0, 1000, size=(2, 16)).astype(np.int32)
    toks, scores = model.beam_decode(dev(torch, prompt), 16, 3)
    assert model.status() == 0
    check_beams(cfg, bf16_round(model.get_params()), prompt, toks.cpu().numpy(), scores.cpu().numpy(), 3)


def test_beam_argument_errors(torch):
    from scratch_decoder_only_b200.gpt import GPT, GPTError
    model = GPT(FP32_64, 17)
    prompt = dev(torch, np.zeros((2, 4), np.int32))
    for W in (0, 9):
        with pytest.raises(GPTError):
            model.beam_decode(prompt, 4, W)
    with pytest.raises(GPTError):
        model.beam_decode(prompt, 4, 5)      # 2 x 5 rows > max_batch 8
    with pytest.raises(GPTError):
        model.beam_decode(prompt, 46, 2)     # 4 + 46 - 1 > max_seq 48
    toks, _ = model.beam_decode(prompt, 4, 4)
    assert model.status() == 0 and toks.shape == (2, 4, 4)
