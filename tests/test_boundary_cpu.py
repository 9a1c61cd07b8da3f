"""Host-side tests of the C ABI and the binding (no GPU needed).

The library must load on a machine without a CUDA driver, export every
entry point include/gpt.h declares, reject bad arguments before touching the
device, and report a CUDA error (not crash) when no device exists.
"""
import ctypes
import os
import re

import numpy as np
import pytest

from scratch_decoder_only_b200 import configs as CF
from scratch_decoder_only_b200 import gpt as G
from scratch_decoder_only_b200 import synthetic as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gpt.h")


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gpt_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from scratch_decoder_only_b200 import build
    if not os.path.exists(G.LIB_PATH):
        build.build()
    return G.load_library()


def test_library_exports_every_declared_symbol(lib):
    names = header_functions()
    assert len(names) >= 20
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(G.EXPORTED) == names


def test_library_has_no_driver_link_dependency():
    # cudart is linked statically and the driver is reached lazily, so the
    # library loads on a host without libcuda (it still fails loudly at the
    # first CUDA call there).
    import subprocess
    out = subprocess.run(["ldd", G.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out and "libcudart" not in out


def test_struct_sizes_match_header():
    assert ctypes.sizeof(G.gpt_config) == 17 * 4
    assert ctypes.sizeof(G.gpt_adamw) == 6 * 4
    assert ctypes.sizeof(G.gpt_scalars) == 7 * 4
    assert ctypes.sizeof(G.gpt_lr_schedule) == 5 * 4


def test_header_is_plain_c_and_matches_the_binding(tmp_path):
    """include/gpt.h compiles as C99 on its own, and every struct's size and
    field offsets seen by a C compiler equal the ctypes mirrors'."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    structs = {"gpt_config": G.gpt_config, "gpt_adamw": G.gpt_adamw, "gpt_scalars": G.gpt_scalars,
               "gpt_lr_schedule": G.gpt_lr_schedule, "gpt_sampling": G.gpt_sampling,
               "gpt_prof_entry": G.gpt_prof_entry}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "gpt.h"', "int main(void) {"]
    for sname, cls in structs.items():
        lines.append(f'  printf("{sname} size %zu\\n", sizeof({sname}));')
        for fname, _ in cls._fields_:
            lines.append(f'  printf("{sname} {fname} %zu\\n", offsetof({sname}, {fname}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                        "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    got = {}
    for ln in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.splitlines():
        parts = ln.split()
        got[tuple(parts[:-1])] = int(parts[-1])
    for sname, cls in structs.items():
        assert got[(sname, "size")] == ctypes.sizeof(cls), sname
        for fname, _ in cls._fields_:
            assert got[(sname, fname)] == getattr(cls, fname).offset, (sname, fname)


def _create(lib, **over):
    mc = CF.TINY_BYTE.model
    cfg = G.make_config(mc)
    for k, v in over.items():
        setattr(cfg, k, v)
    h = ctypes.c_void_p()
    rc = lib.gpt_create(ctypes.byref(cfg), 42, ctypes.byref(h))
    return rc, h


@pytest.mark.parametrize("field,value", [("d_model", 100), ("n_heads", 3), ("d_mlp", 0), ("n_layers", 0),
                                         ("vocab_padded", 10), ("precision", 7), ("max_batch", 0),
                                         ("d_model", 2048)])
def test_create_rejects_bad_config(lib, field, value):
    rc, h = _create(lib, **{field: value})
    assert rc == G.GPT_ERR_ARG and not h.value
    assert lib.gpt_last_error(None).decode()


def test_create_without_device_reports_cuda_error(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device exists")
    rc, h = _create(lib)
    assert rc == G.GPT_ERR_CUDA and not h.value


def test_null_handles_rejected(lib):
    assert lib.gpt_backward(None) == G.GPT_ERR_ARG
    assert lib.gpt_forward_loss(None, None, None, None, 1, 1, None) == G.GPT_ERR_ARG
    assert lib.gpt_status(None) == G.GPT_ERR_ARG
    assert lib.gpt_set_stream(None, None) == G.GPT_ERR_ARG
    n = ctypes.c_size_t()
    assert lib.gpt_num_params(None, ctypes.byref(n)) == G.GPT_ERR_ARG
    lib.gpt_destroy(None)


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(G, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        G.load_library(str(tmp_path / "nope.so"))


# ---- input generators (shared by the oracle and the library; no model arithmetic)

def test_packed_inputs_follow_recipe():
    tok, tgt, seg = S.make_batch(CF.PACKED_SMALL)
    assert tok.shape == (8, 512) and seg.shape == (8, 512)
    assert tok.dtype == np.int32 and tok.min() >= 0 and tok.max() < 8000
    for r in range(8):
        assert seg[r, 0] == 0 and np.all(np.diff(seg[r]) >= 0)
        bounds = np.nonzero(np.diff(seg[r]))[0]
        # every target that crosses a document boundary is ignored
        assert np.all(tgt[r, bounds] == -1)
        lens = np.diff(np.concatenate([[0], bounds + 1, [512]]))
        assert np.all(lens[:-1] >= 16) and np.all(lens <= 512)
    # Zipf(1.1): id 0 is the most frequent
    counts = np.bincount(tok.reshape(-1), minlength=8000)
    assert counts[0] == counts.max()


def test_uniform_and_skewed_bytes():
    tok, tgt, seg = S.make_batch(CF.TINY_BYTE)
    assert tok.shape == (4, 80) and seg is None
    assert np.array_equal(tok[:, 1:], tgt[:, :-1])
    assert tok.max() <= 256
    tok3, _, _ = S.make_batch(CF.BYTE_30M, batch=2)
    frac_printable = np.mean((tok3 >= 32) & (tok3 <= 126))
    assert 0.85 < frac_printable < 0.97
    assert tok3.max() <= 255


def test_generators_are_deterministic():
    a = S.make_batch(CF.GPT2_124M, batch=2, seq=64)
    b = S.make_batch(CF.GPT2_124M, batch=2, seq=64)
    assert all(np.array_equal(x, y) for x, y in zip(a[:2], b[:2]))
