"""GPU tests of the training loop around the step: the device-side
learning-rate schedule, the multi-step call and the loss scaler's growth.

* Cosine schedule with warm-up and a floor ("LucilleAI", "Getting started":
  --lr-scheduler cosine --warmup-steps --min-lr): the optimiser alone, both
  sides given the same fp32 gradients, over steps that cross the warm-up, the
  decay and the floor; every step's weights against the oracle with its
  lr_at(s).
* gpt_train_steps: three steps of the tiny byte model in one call against
  the oracle's three-step trajectory (fp32 bars).
* GradScaler growth ("LucilleAI", "Architecture": GradScaler): a finite step
  taken with 1999 good steps behind it doubles the scale; a non-finite one
  halves it and resets the count.
* Gradient accumulation over micro-batches with a loss weight.
* gpt_train_step, the training step as one replayed CUDA graph, against the
  three separate calls.
"""
import numpy as np
import pytest

from oracle import gpt_oracle as O
from scratch_decoder_only_b200 import configs as CF
from scratch_decoder_only_b200 import synthetic as S
from tests.helpers import ocfg, rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch as t
    assert t.cuda.is_available()
    return t


def dev(torch, a):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()


def test_cosine_schedule_on_device(torch):
    from scratch_decoder_only_b200.gpt import GPT, GPT_LR_COSINE
    wl = CF.TINY_BYTE
    model = GPT(wl.model, wl.init_seed)
    sched = dict(kind=GPT_LR_COSINE, warmup=2, total=6, max_lr=1e-2, min_lr=1e-3)
    model.set_lr_schedule(GPT_LR_COSINE, sched["warmup"], sched["total"], sched["max_lr"], sched["min_lr"])
    hp = CF.AdamWConfig(lr=123.0, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, clip_norm=1e9)
    p = model.get_params().astype(np.float64)
    m = np.zeros_like(p)
    v = np.zeros_like(p)
    rng = np.random.default_rng(8)
    for s in range(9):
        g = rng.normal(0, 1e-3, p.size).astype(np.float32)
        model.set_grads(g)
        model.clip_adamw_step(hp)
        lr = O.lr_at(s, **sched)
        p, m, v, _, _ = O.clip_adamw_step(p, g.astype(np.float64), m, v, s + 1, lr, hp.beta1, hp.beta2, hp.eps,
                                          hp.weight_decay, hp.clip_norm)
        got = model.get_params()
        assert np.max(np.abs(got - p)) <= 1e-6 + 2e-6 * (s + 1), (s, np.max(np.abs(got - p)))
        assert rel(model.scalars()["last_lr"], lr) <= 1e-6, (s, model.scalars()["last_lr"], lr)
    # cleared: the host learning rate applies again
    model.set_lr_schedule(None)
    model.set_grads(rng.normal(0, 1e-3, p.size).astype(np.float32))
    model.clip_adamw_step(CF.AdamWConfig(lr=5e-4, clip_norm=1.0))
    assert model.scalars()["last_lr"] == pytest.approx(5e-4, rel=1e-6)
    assert model.status() == 0


def test_train_steps_matches_oracle_trajectory(torch):
    wl = CF.TINY_BYTE
    cfg = ocfg(wl.model)
    from scratch_decoder_only_b200.gpt import GPT
    K = 3
    batches = [S.make_batch(wl, batch=2, seq=64, seed=wl.data_seed + k) for k in range(K)]
    tok = np.stack([b[0] for b in batches])
    tgt = np.stack([b[1] for b in batches])
    model = GPT(wl.model, wl.init_seed)
    p = model.get_params().astype(np.float64)
    losses = torch.zeros(K, dtype=torch.float32, device="cuda")
    norms = torch.zeros(K, dtype=torch.float32, device="cuda")
    skipped = torch.ones(K, dtype=torch.int32, device="cuda")
    model.train_steps(dev(torch, tok), dev(torch, tgt), None, wl.adamw, losses, norms, skipped)
    assert model.status() == 0
    hp = wl.adamw
    m = np.zeros_like(p)
    v = np.zeros_like(p)
    for k in range(K):
        loss, g = O.loss_and_grads(cfg, p, tok[k], tgt[k])
        p, m, v, norm, sk = O.clip_adamw_step(p, g, m, v, k + 1, hp.lr, hp.beta1, hp.beta2, hp.eps,
                                              hp.weight_decay, hp.clip_norm)
        assert rel(losses[k].item(), loss) <= 1e-4, (k, losses[k].item(), loss)
        assert rel(norms[k].item(), norm) <= 1e-4, (k, norms[k].item(), norm)
        assert int(skipped[k].item()) == 0
    assert model.scalars()["step"] == K
    # each step moves a weight by at most about lr: the trajectories stay close
    assert np.max(np.abs(model.get_params() - p)) <= 2 * hp.lr * K


def test_loss_scale_growth_after_2000_good_steps(torch):
    from scratch_decoder_only_b200.gpt import GPT
    wl = CF.PACKED_SMALL
    model = GPT(wl.model, wl.init_seed)
    rng = np.random.default_rng(9)
    n = model.n_params
    scale = model.scalars()["loss_scale"]
    model.set_scalars(good_steps=1999)
    model.set_grads(rng.normal(0, 1e-3, n).astype(np.float32) * np.float32(scale))
    model.clip_adamw_step(wl.adamw)
    s = model.scalars()
    assert s["loss_scale"] == 2 * scale and s["good_steps"] == 0 and s["last_skipped"] == 0
    # a finite step below the interval only counts
    model.set_grads(rng.normal(0, 1e-3, n).astype(np.float32) * np.float32(2 * scale))
    model.clip_adamw_step(wl.adamw)
    s = model.scalars()
    assert s["loss_scale"] == 2 * scale and s["good_steps"] == 1
    # a non-finite step halves the scale, resets the count and is skipped
    g = rng.normal(0, 1e-3, n).astype(np.float32)
    g[7] = np.inf
    model.set_grads(g)
    model.clip_adamw_step(wl.adamw)
    s = model.scalars()
    assert s["loss_scale"] == scale and s["good_steps"] == 0 and s["last_skipped"] == 1
    # the oracle's rule gives the same sequence
    sc, good = scale, 1999
    sc, good, skip = O.loss_scale_update(sc, good, True)
    assert (sc, good, skip) == (2 * scale, 0, False)
    sc, good, skip = O.loss_scale_update(sc, good, True)
    sc, good, skip = O.loss_scale_update(sc, good, False)
    assert (sc, good, skip) == (scale, 0, True)
    assert model.status() == 0


@pytest.mark.parametrize("wl_name", ["tiny", "packed"])
def test_gradient_accumulation_equals_one_large_batch(torch, wl_name):
    """k = 4 micro-batches with loss weight 1/4 (one gpt_backward, three
    accumulating) give the gradient of the mean loss over the 4x batch: the
    same as one backward over the concatenated batch and as the oracle's
    gradient on it (fp32: rel-L2 1e-3 per tensor; bf16 packed model with loss
    scale 2^15: 3e-2).  Equal weights are exact when every micro-batch has the
    same number of valid targets: each packed row here holds two documents,
    so each has 255 of its 256 targets valid."""
    from scratch_decoder_only_b200.gpt import GPT
    from tests.helpers import per_tensor_rel_l2
    if wl_name == "tiny":
        wl, bar = CF.TINY_BYTE, 1e-3
        mc = wl.model
        tok, tgt, _ = S.make_batch(wl, batch=4, seq=48)
        seg = None
    else:
        wl, bar = CF.PACKED_SMALL, 3e-2
        mc = wl.model
        rng = np.random.default_rng(10)
        x = rng.integers(0, mc.vocab, size=(4, 257))
        segf = np.zeros((4, 257), np.int64)
        for r, cut in enumerate((40, 100, 170, 230)):
            segf[r, cut:] = 1
        tok, tgt = S.shift_targets(x, segf)
        tok, tgt = tok.astype(np.int32), tgt.astype(np.int32)
        seg = segf[:, :256].astype(np.int32)
    cfg = ocfg(mc)
    model = GPT(mc, wl.init_seed)
    p0 = model.get_params()
    scale = model.scalars()["loss_scale"]
    model.set_loss_weight(0.25)
    for k in range(4):
        sl = slice(k, k + 1)
        model.forward_loss(dev(torch, tok[sl]), dev(torch, tgt[sl]), None if seg is None else dev(torch, seg[sl]))
        model.backward(accumulate=k > 0)
    g_acc = model.get_grads() / np.float32(scale)
    model.set_loss_weight(1.0)
    model.forward_loss(dev(torch, tok), dev(torch, tgt), None if seg is None else dev(torch, seg))
    model.backward()
    g_big = model.get_grads() / np.float32(scale)
    assert model.status() == 0
    _, g_ref = O.loss_and_grads(cfg, p0.astype(np.float64), tok, tgt, seg)
    for got in (g_acc, g_big):
        errs = per_tensor_rel_l2(cfg, got, g_ref)
        worst = max(errs, key=errs.get)
        assert errs[worst] <= bar, (worst, errs[worst])
    errs = per_tensor_rel_l2(cfg, g_acc, g_big.astype(np.float64))
    assert max(errs.values()) <= bar


def test_graph_step_matches_three_calls(torch):
    """gpt_train_step (one captured graph per call signature, replayed) leaves
    what gpt_forward_loss + gpt_backward + gpt_clip_adamw_step leave, to the
    rounding that the embedding gradients' atomic order allows: parameters,
    Adam moments, losses and gradient norms after four steps, with
    new tokens written into the captured buffers between replays, a second
    buffer pair (a new capture) and a changed learning rate (another)."""
    from scratch_decoder_only_b200.gpt import GPT
    wl = CF.BYTE_30M
    mc = CF.ModelConfig(**{**wl.model.as_dict(), "n_layers": 2, "max_batch": 2, "max_seq": 256})
    hp = CF.AdamWConfig(lr=3e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, clip_norm=1.0)
    hp2 = CF.AdamWConfig(lr=1e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, clip_norm=1.0)
    a, b = GPT(mc, 11), GPT(mc, 11)
    rng = np.random.default_rng(12)
    batches = [rng.integers(0, mc.vocab, size=(2, 129)).astype(np.int32) for _ in range(4)]
    tok_a, tgt_a = torch.zeros((2, 128), dtype=torch.int32, device="cuda"), torch.zeros((2, 128), dtype=torch.int32,
                                                                                       device="cuda")
    tok_c, tgt_c = tok_a.clone(), tgt_a.clone()
    la, lb = torch.zeros(4, device="cuda"), torch.zeros(4, device="cuda")
    ga, gb = torch.zeros(4, device="cuda"), torch.zeros(4, device="cuda")
    for i, x in enumerate(batches):
        ta, tg = (tok_a, tgt_a) if i != 2 else (tok_c, tgt_c)
        ta.copy_(torch.from_numpy(x[:, :-1])); tg.copy_(torch.from_numpy(x[:, 1:]))
        h = hp if i < 3 else hp2
        a.train_step(ta, tg, None, h, la[i:i + 1], ga[i:i + 1])
        b.forward_loss(ta, tg, None, lb[i:i + 1])
        b.backward()
        b.clip_adamw_step(h, gb[i:i + 1])
    torch.cuda.synchronize()
    assert a.status() == 0 and b.status() == 0
    # losses and norms see the embedding rows, so they match to rounding
    assert np.allclose(la.cpu().numpy(), lb.cpu().numpy(), rtol=1e-5, atol=0)
    assert np.allclose(ga.cpu().numpy(), gb.cpu().numpy(), rtol=1e-5, atol=0)
    # the embedding tables (token rows, then positions: the first
    # (Vp + max_seq) C values) take their gradients by atomic scatter-add, whose
    # order varies from run to run, and every later step sees them: the
    # parameters and moments agree to rounding (their update is one fused pass
    # over the same gradients, so a graph that dropped, repeated or reordered a
    # kernel would differ by whole steps, not by rounding)
    for ga_, gb_ in ((a.get_params(), b.get_params()), (a.get_adam_m(), b.get_adam_m()),
                     (a.get_adam_v(), b.get_adam_v())):
        assert np.allclose(ga_, gb_, rtol=1e-3, atol=1e-7), np.max(np.abs(ga_ - gb_))
