"""FP16 AMP: fp16 GEMM and attention operands and activations with fp32
accumulation, fp32 master weights and a dynamic loss scale ("LucilleAI",
"Architecture (from source)": autocast FP16 + GradScaler; "Real measured
numbers": Tensor-Core AMP in FP16), against the fp64 oracle with the 16-bit
bars (loss rel 1e-2, per-tensor gradient rel-L2 3e-2, weights after one step
within 1e-3).

* the packed model (head size 32, block-diagonal attention) at its full
  8 x 512 size, loss scale 2^15;
* a GPT-2-shaped model at head size 64 (the tcgen05 attention and GEMM
  kernels with fp16 operands), plain and packed;
* gradient accumulation in fp16 (4 micro-batches equal one 4x batch);
* greedy decoding in fp16 against the oracle's logits for the generated
  sequence.
"""
import numpy as np
import pytest

from oracle import gpt_oracle as O
from scratch_decoder_only_b200 import configs as CF
from scratch_decoder_only_b200 import synthetic as S
from tests.helpers import ocfg, per_tensor_rel_l2, rel, tame_attention

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch as t
    assert t.cuda.is_available()
    return t


def dev(torch, a):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()


def fp16_model(mc):
    return CF.ModelConfig(**{**mc.as_dict(), "precision": "fp16", "loss_scaling": True, "init_loss_scale": 2.0 ** 15})


def step_and_compare(torch, mc, tok, tgt, seg, hp, seed=42):
    from scratch_decoder_only_b200.gpt import GPT
    cfg = ocfg(mc)
    model = GPT(mc, seed)
    p0 = model.get_params()
    loss = torch.zeros(1, dtype=torch.float32, device="cuda")
    model.forward_loss(dev(torch, tok), dev(torch, tgt), dev(torch, seg), loss)
    scale = model.scalars()["loss_scale"]
    model.backward()
    g = model.get_grads() / np.float32(scale)
    sk = torch.zeros(1, dtype=torch.int32, device="cuda")
    model.clip_adamw_step(hp, None, sk)
    p1 = model.get_params()
    assert model.status() == 0, model.last_error()
    assert int(sk.item()) == 0
    ref_loss, ref_g = O.loss_and_grads(cfg, p0.astype(np.float64), tok, tgt, seg)
    assert rel(loss.item(), ref_loss) <= 1e-2, (loss.item(), ref_loss)
    errs = per_tensor_rel_l2(cfg, g, ref_g)
    worst = max(errs, key=errs.get)
    assert errs[worst] <= 3e-2, (worst, errs[worst])
    ref_p1, _, _, _, _ = O.clip_adamw_step(p0.astype(np.float64), ref_g, np.zeros(p0.size), np.zeros(p0.size), 1,
                                           hp.lr, hp.beta1, hp.beta2, hp.eps, hp.weight_decay, hp.clip_norm)
    d = np.abs(p1 - ref_p1)
    flips = np.sign(g) != np.sign(ref_g)
    assert np.max(d[~flips]) <= 1e-3
    assert np.max(d) <= 2 * hp.lr + 1e-6
    return errs[worst]


def test_fp16_packed_model_full_size(torch):
    wl = CF.PACKED_SMALL
    mc = fp16_model(wl.model)
    tok, tgt, seg = S.make_batch(wl)
    worst = step_and_compare(torch, mc, tok, tgt, seg, wl.adamw)
    print(f"fp16 packed: worst per-tensor rel-L2 {worst:.2e}")


@pytest.mark.parametrize("packed", [False, True])
def test_fp16_head64_tensor_core_path(torch, packed):
    mc = CF.ModelConfig(vocab=1000, vocab_padded=1024, d_model=256, n_heads=4, d_mlp=1024, n_layers=2,
                        max_seq=512, max_batch=2, tied=True, precision="fp16", loss_scaling=True,
                        init_loss_scale=2.0 ** 15)
    rng = np.random.default_rng(40)
    x = rng.integers(0, 1000, size=(2, 385))
    seg = None
    if packed:
        seg = np.zeros((2, 385), np.int64)
        seg[0, 150:] = 1
        seg[1, 300:] = 1
    tok, tgt = S.shift_targets(x, seg)
    seg_in = None if seg is None else seg[:, :384].astype(np.int32)
    worst = step_and_compare(torch, mc, tok.astype(np.int32), tgt.astype(np.int32), seg_in,
                             CF.AdamWConfig(lr=3e-4, clip_norm=1.0))
    print(f"fp16 d=64 packed={packed}: worst per-tensor rel-L2 {worst:.2e}")


def test_fp16_gradient_accumulation(torch):
    from scratch_decoder_only_b200.gpt import GPT
    mc = CF.ModelConfig(vocab=1000, vocab_padded=1024, d_model=256, n_heads=4, d_mlp=1024, n_layers=2,
                        max_seq=256, max_batch=4, tied=False, precision="fp16", loss_scaling=True,
                        init_loss_scale=2.0 ** 15)
    rng = np.random.default_rng(41)
    tok, tgt = S.random_tokens(rng, 4, 256, 1000)
    cfg = ocfg(mc)
    model = GPT(mc, 3)
    p0 = model.get_params()
    scale = model.scalars()["loss_scale"]
    model.set_loss_weight(0.25)
    for k in range(4):
        model.forward_loss(dev(torch, tok[k:k + 1]), dev(torch, tgt[k:k + 1]))
        model.backward(accumulate=k > 0)
    g_acc = model.get_grads() / np.float32(scale)
    assert model.status() == 0
    _, g_ref = O.loss_and_grads(cfg, p0.astype(np.float64), tok, tgt)
    errs = per_tensor_rel_l2(cfg, g_acc, g_ref)
    assert max(errs.values()) <= 3e-2, max(errs, key=errs.get)


def test_fp16_greedy_decode_against_oracle_logits(torch):
    from scratch_decoder_only_b200.gpt import GPT
    mc = CF.ModelConfig(vocab=1000, vocab_padded=1024, d_model=256, n_heads=4, d_mlp=1024, n_layers=2,
                        max_seq=64, max_batch=2, tied=False, precision="fp16", init_std=0.3)
    cfg = ocfg(mc)
    model = GPT(mc, 13)
    tame_attention(model, cfg)
    rng = np.random.default_rng(42)
    Tp, n_new = 12, 16
    prompt = rng.integers(0, 1000, size=(2, Tp)).astype(np.int32)
    out = model.greedy_decode(dev(torch, prompt), n_new).cpu().numpy()
    assert model.status() == 0
    p32 = model.get_params()
    pw = p32.astype(np.float16).astype(np.float64)       # the fp16 working copy
    seq = np.concatenate([prompt, out[:, :-1]], axis=1)
    z, _ = O.forward(cfg, pw, seq)
    z = z.reshape(2, Tp + n_new - 1, -1)[:, Tp - 1:, :1000]
    top = z.max(axis=2)
    picked = np.take_along_axis(z, out[:, :, None].astype(np.int64), axis=2)[:, :, 0]
    assert np.all(top - picked <= 0.01 * np.abs(z).max(axis=2))
