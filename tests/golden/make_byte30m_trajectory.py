"""Write the oracle's 20-step AdamW trajectory of the byte-level 30M model.

Calls only the oracle (and the seeded input generator): the stored values are
the oracle's, never the CUDA path's.  Workload: the byte-level ~30M-parameter
GPT (vocab 257, d_model 512, 8 heads x 64, MLP 2048, 8 blocks) at 4 rows x
1024 tokens per step (the reduced batch the 20-step trajectory is run at, so
that the fp64 oracle finishes in minutes), AdamW lr 3e-4, betas (0.9, 0.999),
eps 1e-8, wd 0.01, clip 1.0 ("Smallem", "Ce qu'est un modele de langage": a
30M-parameter byte-level network; AdamW with decoupled decay as in "Feste",
"Manual Backpropagation from scratch"; global L2 clip as in "RustGPT",
"Technical implementation").  Step s draws its batch from seed 103 + s.

Output (JSON): per-step loss and unscaled global gradient norm, and for 4096
fixed parameter indices the initial and final fp32-master values.

    python tests/golden/make_byte30m_trajectory.py [out.json]
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import gpt_oracle as O  # noqa: E402
from scratch_decoder_only_b200 import configs as CF  # noqa: E402
from scratch_decoder_only_b200 import synthetic as S  # noqa: E402

STEPS, BATCH, SEQ, N_SAMPLE = 20, 4, 1024, 4096


def main(out_path):
    wl = CF.BYTE_30M
    mc = wl.model
    cfg = O.OracleConfig(vocab=mc.vocab, vocab_padded=mc.vocab_padded, d_model=mc.d_model, n_heads=mc.n_heads,
                         d_mlp=mc.d_mlp, n_layers=mc.n_layers, max_seq=mc.max_seq, tied=mc.tied,
                         ln_eps=mc.ln_eps, init_std=mc.init_std)
    hp = wl.adamw
    p0 = O.init_params(cfg, wl.init_seed).astype(np.float64)
    p, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
    losses, norms = [], []
    for s in range(STEPS):
        tok, tgt, seg = S.make_batch(wl, batch=BATCH, seq=SEQ, seed=wl.data_seed + s)
        loss, g = O.loss_and_grads(cfg, p, tok, tgt, seg, np.float64)
        p, m, v, norm, skipped = O.clip_adamw_step(p, g, m, v, s + 1, hp.lr, hp.beta1, hp.beta2, hp.eps,
                                                   hp.weight_decay, hp.clip_norm)
        assert not skipped
        losses.append(float(loss))
        norms.append(float(norm))
        print(f"step {s}: loss {loss:.6f} norm {norm:.6f}", flush=True)
    idx = np.sort(np.random.default_rng(7).choice(p0.size, N_SAMPLE, replace=False))
    rec = {
        "workload": wl.name, "batch": BATCH, "seq": SEQ, "steps": STEPS, "init_seed": wl.init_seed,
        "data_seeds": [wl.data_seed + s for s in range(STEPS)],
        "adamw": {"lr": hp.lr, "beta1": hp.beta1, "beta2": hp.beta2, "eps": hp.eps,
                  "weight_decay": hp.weight_decay, "clip_norm": hp.clip_norm},
        "loss": losses, "grad_norm": norms,
        "delta_l2_full": float(np.linalg.norm(p - p0)),
        "sample_index": idx.tolist(), "p0": p0[idx].tolist(), "p_final": p[idx].tolist(),
    }
    with open(out_path, "w") as f:
        json.dump(rec, f)


if __name__ == "__main__":
    here = os.path.dirname(os.path.abspath(__file__))
    main(sys.argv[1] if len(sys.argv) > 1 else os.path.join(here, "byte30m_trajectory_b4_t1024_20steps.json"))
