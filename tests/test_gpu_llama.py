"""GPU parity of the Llama-style block against the oracle ("NTransformer"
page, key features: Llama architecture with RoPE, GQA, SwiGLU, KV cache).

RMSNorm, rotary positions applied to q and k after the qkv GEMM (their
inverse to dq and dk), two query heads per key/value head read by the
tcgen05 attention through its column layout (and the per-query-head key/value
gradients summed into the shared heads), SwiGLU between the up and down
GEMMs, no biases.  Bars: loss rel 1e-2, per-tensor gradient rel-L2 3e-2.
"""
import numpy as np
import pytest

from oracle import gpt_oracle as O
from scratch_decoder_only_b200 import configs as CF
from scratch_decoder_only_b200 import synthetic as S
from tests.helpers import ocfg, tame_attention, per_tensor_rel_l2, rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch as t
    assert t.cuda.is_available()
    return t


def dev(torch, a):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()


def llama_cfg(kv=2, precision="bf16", tied=False, max_seq=512, max_batch=2, init_std=0.02):
    return CF.ModelConfig(vocab=1000, vocab_padded=1024, d_model=256, n_heads=4, d_mlp=672, n_layers=2,
                          max_seq=max_seq, max_batch=max_batch, tied=tied, precision=precision, arch="llama",
                          n_kv_heads=kv, init_std=init_std,
                          loss_scaling=precision == "fp16", init_loss_scale=2.0 ** 15 if precision == "fp16" else 1.0)


def test_llama_init_matches_oracle(torch):
    from scratch_decoder_only_b200.gpt import GPT
    mc = llama_cfg()
    model = GPT(mc, 9)
    got = model.get_params()
    want = O.init_params(ocfg(mc), 9)
    assert got.size == want.size == mc.num_params()
    diff = got.view(np.uint32).astype(np.int64) - want.view(np.uint32).astype(np.int64)
    assert np.count_nonzero(diff) <= max(1, got.size // 1_000_000) and np.max(np.abs(diff)) <= 1


@pytest.mark.parametrize("kv,packed,precision,tied", [(2, False, "bf16", False), (2, True, "bf16", False),
                                                     (4, False, "bf16", True), (1, True, "fp16", False)])
def test_llama_step_matches_oracle(torch, kv, packed, precision, tied):
    from scratch_decoder_only_b200.gpt import GPT
    mc = llama_cfg(kv=kv, precision=precision, tied=tied)
    cfg = ocfg(mc)
    rng = np.random.default_rng(50 + kv)
    T = 384
    x = rng.integers(0, 1000, size=(2, T + 1))
    seg = None
    if packed:
        seg = np.zeros((2, T + 1), np.int64)
        seg[0, 100:] = 1
        seg[0, 250:] = 2
        seg[1, 200:] = 1
    tok, tgt = S.shift_targets(x, seg)
    tok, tgt = tok.astype(np.int32), tgt.astype(np.int32)
    seg_in = None if seg is None else seg[:, :T].astype(np.int32)
    model = GPT(mc, 11)
    p0 = model.get_params()
    loss = torch.zeros(1, dtype=torch.float32, device="cuda")
    model.forward_loss(dev(torch, tok), dev(torch, tgt), dev(torch, seg_in), loss)
    scale = model.scalars()["loss_scale"]
    model.backward()
    g = model.get_grads() / np.float32(scale)
    assert model.status() == 0, model.last_error()
    ref_loss, ref_g = O.loss_and_grads(cfg, p0.astype(np.float64), tok, tgt, seg_in)
    assert rel(loss.item(), ref_loss) <= 1e-2, (loss.item(), ref_loss)
    errs = per_tensor_rel_l2(cfg, g, ref_g)
    worst = max(errs, key=errs.get)
    assert errs[worst] <= 3e-2, (worst, errs[worst], errs)
    print(f"llama kv={kv} packed={packed} {precision}: worst per-tensor rel-L2 {errs[worst]:.2e} ({worst})")


def test_llama_mask_bit_identity(torch):
    """A changed token leaves every earlier position's logits bit-identical."""
    from scratch_decoder_only_b200.gpt import GPT
    mc = llama_cfg()
    model = GPT(mc, 12)
    rng = np.random.default_rng(53)
    tok = rng.integers(0, 1000, size=(2, 300)).astype(np.int32)
    model.forward_loss(dev(torch, tok))
    base = model.get_logits(2, 300).reshape(2, 300, -1)
    t2 = tok.copy()
    t2[:, 170] = (t2[:, 170] + 3) % 1000
    model.forward_loss(dev(torch, t2))
    alt = model.get_logits(2, 300).reshape(2, 300, -1)
    assert np.array_equal(base[:, :170], alt[:, :170])
    assert not np.array_equal(base[:, 170], alt[:, 170])


@pytest.mark.parametrize("B", [2, 12])
def test_llama_greedy_decode_against_oracle_logits(torch, B):
    """Decoding with the rotated keys in a cache of two key/value heads: each
    generated token is the oracle's argmax for the generated sequence (full
    prefix, no cache) up to a bf16 tolerance of 1 % of the row's logit scale;
    exact where the top-2 gap is clear.  Batch 2 takes the GEMV projections, batch 12 the tensor-core GEMM."""
    from scratch_decoder_only_b200.gpt import GPT
    mc = llama_cfg(max_seq=64, max_batch=12, init_std=0.3)
    cfg = ocfg(mc)
    model = GPT(mc, 14)
    tame_attention(model, cfg)
    rng = np.random.default_rng(54 + B)
    Tp, n_new = 16, 20
    prompt = rng.integers(0, 1000, size=(B, Tp)).astype(np.int32)
    out = model.greedy_decode(dev(torch, prompt), n_new).cpu().numpy()
    assert model.status() == 0
    p32 = model.get_params()
    u = p32.view(np.uint32)
    pb = ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).view(np.float32).astype(np.float64)
    seq = np.concatenate([prompt, out[:, :-1]], axis=1)
    z, _ = O.forward(cfg, pb, seq)
    z = z.reshape(B, Tp + n_new - 1, -1)[:, Tp - 1:, :1000]
    top = z.max(axis=2)
    picked = np.take_along_axis(z, out[:, :, None].astype(np.int64), axis=2)[:, :, 0]
    srt = np.sort(z, axis=2)
    gap = srt[:, :, -1] - srt[:, :, -2]
    tol = 0.01 * np.abs(z).max(axis=2)    # 1 % of the row's logit scale (bf16 activations)
    assert np.all(top - picked <= tol), (np.argwhere(top - picked > tol), (top - picked).max())
    clear = gap > tol
    assert clear.mean() >= 0.7
    assert np.array_equal(out[clear], np.argmax(z, axis=2)[clear])
