"""ctypes binding of libgpt.so (include/gpt.h): argument marshalling only.

Every step of the path runs in the library's CUDA kernels; this module passes
device pointers of torch tensors, the current torch stream and plain
structs.  It raises GPTError for any non-zero return code and refuses to
run without the built library (there is no fallback).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .configs import AdamWConfig, ModelConfig

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgpt.so")

GPT_OK = 0
ERR_NAMES = {-1: "GPT_ERR_ARG", -2: "GPT_ERR_STATE", -3: "GPT_ERR_CUDA", -4: "GPT_ERR_TIMEOUT",
             -5: "GPT_ERR_DEVICE", -6: "GPT_ERR_NOMEM"}
GPT_ERR_ARG, GPT_ERR_STATE, GPT_ERR_CUDA, GPT_ERR_TIMEOUT, GPT_ERR_DEVICE, GPT_ERR_NOMEM = -1, -2, -3, -4, -5, -6

EXPORTED = [
    "gpt_create", "gpt_destroy", "gpt_set_stream", "gpt_forward_loss", "gpt_backward",
    "gpt_clip_adamw_step", "gpt_greedy_decode", "gpt_num_params", "gpt_get_params", "gpt_set_params",
    "gpt_get_grads", "gpt_set_grads", "gpt_get_adam_m", "gpt_set_adam_m", "gpt_get_adam_v",
    "gpt_set_adam_v", "gpt_get_logits", "gpt_get_residual", "gpt_get_scalars", "gpt_set_scalars", "gpt_status",
    "gpt_device_error", "gpt_last_error", "gpt_debug_poison_grad", "gpt_debug_wait_timeout",
    "gpt_kernel_launches", "gpt_profile_enable", "gpt_profile_read", "gpt_gemm_bf16",
    "gpt_gemm_bf16_splitk_noalloc", "gpt_noalloc_status", "gpt_set_lr_schedule", "gpt_train_steps",
    "gpt_sample_decode", "gpt_backward_accumulate", "gpt_set_loss_weight", "gpt_beam_decode", "gpt_train_step",
]


class GPTError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{ERR_NAMES.get(code, code)}: {msg}")
        self.code = code


class gpt_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("vocab", "vocab_padded", "d_model", "n_heads", "d_mlp",
                                              "n_layers", "max_seq", "max_batch", "tied", "precision",
                                              "loss_scaling")] + \
               [("init_loss_scale", ctypes.c_float), ("ln_eps", ctypes.c_float), ("init_std", ctypes.c_float),
                ("arch", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32), ("rope_base", ctypes.c_float)]


class gpt_adamw(ctypes.Structure):
    _fields_ = [(n, ctypes.c_float) for n in ("lr", "beta1", "beta2", "eps", "weight_decay", "clip_norm")]


class gpt_prof_entry(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 24), ("launches", ctypes.c_int32), ("ms", ctypes.c_double),
                ("flops", ctypes.c_double), ("bytes", ctypes.c_double)]


class gpt_scalars(ctypes.Structure):
    _fields_ = [("loss_scale", ctypes.c_float), ("good_steps", ctypes.c_int32), ("step", ctypes.c_int32),
                ("last_loss", ctypes.c_float), ("last_grad_norm", ctypes.c_float),
                ("last_skipped", ctypes.c_int32), ("last_lr", ctypes.c_float)]


GPT_LR_CONSTANT, GPT_LR_COSINE = 0, 1


class gpt_sampling(ctypes.Structure):
    _fields_ = [("temperature", ctypes.c_float), ("top_k", ctypes.c_int32), ("top_p", ctypes.c_float)]


class gpt_lr_schedule(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("warmup_steps", ctypes.c_int32), ("total_steps", ctypes.c_int32),
                ("max_lr", ctypes.c_float), ("min_lr", ctypes.c_float)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libgpt.so and declare every exported signature."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m scratch_decoder_only_b200.build`")
    L = ctypes.CDLL(path)
    P, I, S, F, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float, ctypes.c_uint64
    H = ctypes.c_void_p
    sig = {
        "gpt_create": ([ctypes.POINTER(gpt_config), U64, ctypes.POINTER(H)], I),
        "gpt_destroy": ([H], None),
        "gpt_set_stream": ([H, P], I),
        "gpt_forward_loss": ([H, P, P, P, I, I, P], I),
        "gpt_backward": ([H], I),
        "gpt_backward_accumulate": ([H], I),
        "gpt_set_loss_weight": ([H, F], I),
        "gpt_clip_adamw_step": ([H, ctypes.POINTER(gpt_adamw), P, P], I),
        "gpt_greedy_decode": ([H, P, I, I, I, P], I),
        "gpt_num_params": ([H, ctypes.POINTER(S)], I),
        "gpt_get_logits": ([H, P, S], I),
        "gpt_get_residual": ([H, I, P, S], I),
        "gpt_get_scalars": ([H, ctypes.POINTER(gpt_scalars)], I),
        "gpt_set_scalars": ([H, ctypes.POINTER(gpt_scalars)], I),
        "gpt_status": ([H], I),
        "gpt_device_error": ([H, ctypes.POINTER(ctypes.c_uint32)], I),
        "gpt_last_error": ([H], ctypes.c_char_p),
        "gpt_debug_poison_grad": ([H, S, F], I),
        "gpt_debug_wait_timeout": ([H, I], I),
        "gpt_kernel_launches": ([ctypes.POINTER(ctypes.c_uint64)], I),
        "gpt_profile_enable": ([H, I], I),
        "gpt_gemm_bf16": ([I, I, I, P, ctypes.c_long, I, P, ctypes.c_long, I, P, ctypes.c_long, P], I),
        "gpt_gemm_bf16_splitk_noalloc": ([I, I, I, P, ctypes.c_long, I, P, ctypes.c_long, I, I, P, ctypes.c_long, P],
                                         I),
        "gpt_noalloc_status": ([P], I),
        "gpt_set_lr_schedule": ([H, ctypes.POINTER(gpt_lr_schedule)], I),
        "gpt_sample_decode": ([H, P, I, I, I, ctypes.POINTER(gpt_sampling), P, P], I),
        "gpt_beam_decode": ([H, P, I, I, I, I, P, P], I),
        "gpt_train_steps": ([H, P, P, P, I, I, I, ctypes.POINTER(gpt_adamw), P, P, P], I),
        "gpt_train_step": ([H, P, P, P, I, I, ctypes.POINTER(gpt_adamw), P, P, P], I),
        "gpt_profile_read": ([H, ctypes.POINTER(gpt_prof_entry), I, ctypes.POINTER(I)], I),
    }
    for n in ("params", "grads", "adam_m", "adam_v"):
        sig[f"gpt_get_{n}"] = ([H, P, S], I)
        sig[f"gpt_set_{n}"] = ([H, P, S], I)
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def make_config(mc: ModelConfig) -> gpt_config:
    return gpt_config(vocab=mc.vocab, vocab_padded=mc.vocab_padded, d_model=mc.d_model, n_heads=mc.n_heads,
                      d_mlp=mc.d_mlp, n_layers=mc.n_layers, max_seq=mc.max_seq, max_batch=mc.max_batch,
                      tied=int(mc.tied), precision={"fp32": 0, "bf16": 1, "fp16": 2}[mc.precision],
                      loss_scaling=int(mc.loss_scaling), init_loss_scale=mc.init_loss_scale,
                      ln_eps=mc.ln_eps, init_std=mc.init_std, arch={"gpt2": 0, "llama": 1}[mc.arch],
                      n_kv_heads=mc.n_kv_heads, rope_base=mc.rope_base)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def gemm_bf16(A, B, a_t=False, b_t=False, M=None, N=None, K=None, lda=None, ldb=None):
    """C = A(M x K) . B(N x K)^T on the library's tensor-core GEMM (fp32 C).

    A, B: 2-D bf16 CUDA tensors holding the operands as stored (transposed
    storage when a_t / b_t)."""
    import torch
    L = load_library()
    if M is None:
        M = A.shape[1] if a_t else A.shape[0]
        K = A.shape[0] if a_t else A.shape[1]
        N = B.shape[1] if b_t else B.shape[0]
    lda = lda or A.stride(0)
    ldb = ldb or B.stride(0)
    C = torch.empty((M, N), dtype=torch.float32, device=A.device)
    s = torch.cuda.current_stream().cuda_stream
    rc = L.gpt_gemm_bf16(M, N, K, ctypes.c_void_p(A.data_ptr()), lda, int(a_t), ctypes.c_void_p(B.data_ptr()),
                         ldb, int(b_t), ctypes.c_void_p(C.data_ptr()), N, ctypes.c_void_p(s))
    if rc != GPT_OK:
        raise GPTError(rc, "gpt_gemm_bf16")
    return C


def gemm_bf16_splitk_noalloc(A, B, a_t=False, b_t=False, splits=4, M=None, N=None, K=None, lda=None, ldb=None):
    """Split-K form of gemm_bf16 whose partial sums use the library's fixed
    device scratch array (no device allocation inside the call)."""
    import torch
    L = load_library()
    if M is None:
        M = A.shape[1] if a_t else A.shape[0]
        K = A.shape[0] if a_t else A.shape[1]
        N = B.shape[1] if b_t else B.shape[0]
    lda = lda or A.stride(0)
    ldb = ldb or B.stride(0)
    C = torch.empty((M, N), dtype=torch.float32, device=A.device)
    s = torch.cuda.current_stream().cuda_stream
    rc = L.gpt_gemm_bf16_splitk_noalloc(M, N, K, ctypes.c_void_p(A.data_ptr()), lda, int(a_t),
                                        ctypes.c_void_p(B.data_ptr()), ldb, int(b_t), splits,
                                        ctypes.c_void_p(C.data_ptr()), N, ctypes.c_void_p(s))
    if rc != GPT_OK:
        raise GPTError(rc, L.gpt_last_error(None).decode())
    return C


def noalloc_status():
    """Synchronise the current stream and return (and clear) the no-allocation
    GEMM's sticky status: GPT_OK, or GPT_ERR_TIMEOUT after a wait gave up."""
    import torch
    L = load_library()
    return L.gpt_noalloc_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


class GPT:
    """One model instance on the current CUDA device (a gpt_model handle)."""

    def __init__(self, mc: ModelConfig, seed: int = 42):
        import torch
        self.torch = torch
        self.lib = load_library()
        self.mc = mc
        h = ctypes.c_void_p()
        cfg = make_config(mc)
        rc = self.lib.gpt_create(ctypes.byref(cfg), ctypes.c_uint64(seed), ctypes.byref(h))
        if rc != GPT_OK:
            raise GPTError(rc, self.lib.gpt_last_error(None).decode())
        self.h = h
        n = ctypes.c_size_t()
        self._check(self.lib.gpt_num_params(self.h, ctypes.byref(n)))
        self.n_params = n.value

    # -- plumbing
    def _check(self, rc):
        if rc != GPT_OK:
            raise GPTError(rc, self.lib.gpt_last_error(self.h).decode())
        return rc

    def _sync_stream(self):
        s = self.torch.cuda.current_stream().cuda_stream
        self._check(self.lib.gpt_set_stream(self.h, ctypes.c_void_p(s)))

    def close(self):
        if getattr(self, "h", None):
            self.lib.gpt_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- the step
    def forward_loss(self, tokens, targets=None, seg_ids=None, loss=None):
        B, T = tokens.shape
        self._sync_stream()
        return self._check(self.lib.gpt_forward_loss(self.h, _ptr(tokens), _ptr(targets), _ptr(seg_ids),
                                                     B, T, _ptr(loss)))

    def backward(self, accumulate=False):
        self._sync_stream()
        if accumulate:
            return self._check(self.lib.gpt_backward_accumulate(self.h))
        return self._check(self.lib.gpt_backward(self.h))

    def set_loss_weight(self, w):
        self._sync_stream()
        return self._check(self.lib.gpt_set_loss_weight(self.h, w))

    def clip_adamw_step(self, hp: AdamWConfig, grad_norm=None, skipped=None):
        self._sync_stream()
        a = gpt_adamw(lr=hp.lr, beta1=hp.beta1, beta2=hp.beta2, eps=hp.eps, weight_decay=hp.weight_decay,
                      clip_norm=hp.clip_norm)
        return self._check(self.lib.gpt_clip_adamw_step(self.h, ctypes.byref(a), _ptr(grad_norm), _ptr(skipped)))

    def set_lr_schedule(self, kind=GPT_LR_COSINE, warmup_steps=0, total_steps=1, max_lr=0.0, min_lr=0.0):
        """Device-side learning-rate schedule (kind None clears it)."""
        self._sync_stream()
        if kind is None:
            return self._check(self.lib.gpt_set_lr_schedule(self.h, None))
        sch = gpt_lr_schedule(kind=kind, warmup_steps=warmup_steps, total_steps=total_steps, max_lr=max_lr,
                              min_lr=min_lr)
        return self._check(self.lib.gpt_set_lr_schedule(self.h, ctypes.byref(sch)))

    def train_steps(self, tokens, targets, seg_ids, hp: AdamWConfig, losses=None, grad_norms=None, skipped=None):
        """K steps over tokens / targets / seg_ids of shape [K, B, T], one call."""
        K, B, T = tokens.shape
        self._sync_stream()
        a = gpt_adamw(lr=hp.lr, beta1=hp.beta1, beta2=hp.beta2, eps=hp.eps, weight_decay=hp.weight_decay,
                      clip_norm=hp.clip_norm)
        return self._check(self.lib.gpt_train_steps(self.h, _ptr(tokens), _ptr(targets), _ptr(seg_ids), K, B, T,
                                                    ctypes.byref(a), _ptr(losses), _ptr(grad_norms),
                                                    _ptr(skipped)))

    def greedy_decode(self, prompt, n_new, out=None):
        B, Tp = prompt.shape
        if out is None:
            out = self.torch.empty((B, n_new), dtype=self.torch.int32, device=prompt.device)
        self._sync_stream()
        self._check(self.lib.gpt_greedy_decode(self.h, _ptr(prompt), B, Tp, n_new, _ptr(out)))
        return out

    def sample_decode(self, prompt, n_new, uniforms, temperature=1.0, top_k=0, top_p=1.0, out=None):
        """Sampled continuation; uniforms: device float32 [B, n_new] in [0, 1)."""
        B, Tp = prompt.shape
        if out is None:
            out = self.torch.empty((B, n_new), dtype=self.torch.int32, device=prompt.device)
        sp = gpt_sampling(temperature=temperature, top_k=top_k, top_p=top_p)
        self._sync_stream()
        self._check(self.lib.gpt_sample_decode(self.h, _ptr(prompt), B, Tp, n_new, ctypes.byref(sp), _ptr(uniforms),
                                               _ptr(out)))
        return out

    def beam_decode(self, prompt, n_new, width):
        """Beam search: returns (tokens int32 [B, width, n_new], scores float32
        [B, width]) on the prompt's device, beams best first."""
        B, Tp = prompt.shape
        out = self.torch.empty((B, width, n_new), dtype=self.torch.int32, device=prompt.device)
        scores = self.torch.empty((B, width), dtype=self.torch.float32, device=prompt.device)
        self._sync_stream()
        self._check(self.lib.gpt_beam_decode(self.h, _ptr(prompt), B, Tp, n_new, width, _ptr(out), _ptr(scores)))
        return out, scores

    # -- state access (synchronous)
    def _get(self, which, dst=None):
        if dst is None:
            dst = np.empty(self.n_params, dtype=np.float32)
        p = ctypes.c_void_p(dst.ctypes.data) if isinstance(dst, np.ndarray) else _ptr(dst)
        self._sync_stream()
        self._check(getattr(self.lib, f"gpt_get_{which}")(self.h, p, self.n_params))
        return dst

    def _set(self, which, src):
        src = np.ascontiguousarray(src, dtype=np.float32) if isinstance(src, np.ndarray) else src
        p = ctypes.c_void_p(src.ctypes.data) if isinstance(src, np.ndarray) else _ptr(src)
        self._sync_stream()
        self._check(getattr(self.lib, f"gpt_set_{which}")(self.h, p, self.n_params))

    def get_params(self, dst=None): return self._get("params", dst)
    def set_params(self, src): self._set("params", src)
    def get_grads(self, dst=None): return self._get("grads", dst)
    def set_grads(self, src): self._set("grads", src)
    def get_adam_m(self, dst=None): return self._get("adam_m", dst)
    def set_adam_m(self, src): self._set("adam_m", src)
    def get_adam_v(self, dst=None): return self._get("adam_v", dst)
    def set_adam_v(self, src): self._set("adam_v", src)

    def get_logits(self, B, T):
        out = np.empty((B * T, self.mc.vocab_padded), dtype=np.float32)
        self._sync_stream()
        self._check(self.lib.gpt_get_logits(self.h, ctypes.c_void_p(out.ctypes.data), out.size))
        return out

    def get_residual(self, layer, B, T):
        out = np.empty((B * T, self.mc.d_model), dtype=np.float32)
        self._sync_stream()
        self._check(self.lib.gpt_get_residual(self.h, layer, ctypes.c_void_p(out.ctypes.data), out.size))
        return out

    def scalars(self) -> dict:
        s = gpt_scalars()
        self._check(self.lib.gpt_get_scalars(self.h, ctypes.byref(s)))
        return {k: getattr(s, k) for k, _ in gpt_scalars._fields_}

    def set_scalars(self, **kw):
        s = gpt_scalars()
        self._check(self.lib.gpt_get_scalars(self.h, ctypes.byref(s)))
        for k, v in kw.items():
            setattr(s, k, v)
        self._check(self.lib.gpt_set_scalars(self.h, ctypes.byref(s)))

    def status(self) -> int:
        return self.lib.gpt_status(self.h)

    def device_error(self) -> int:
        b = ctypes.c_uint32()
        self._check(self.lib.gpt_device_error(self.h, ctypes.byref(b)))
        return b.value

    def last_error(self) -> str:
        return self.lib.gpt_last_error(self.h).decode()

    def kernel_launches(self) -> int:
        n = ctypes.c_uint64()
        self._check(self.lib.gpt_kernel_launches(ctypes.byref(n)))
        return n.value

    def profile_enable(self, on=True):
        self._sync_stream()
        self._check(self.lib.gpt_profile_enable(self.h, int(on)))

    def profile_read(self) -> dict:
        arr = (gpt_prof_entry * 16)()
        n = ctypes.c_int()
        self._check(self.lib.gpt_profile_read(self.h, arr, 16, ctypes.byref(n)))
        return {arr[i].name.decode(): {"launches": arr[i].launches, "ms": arr[i].ms, "flops": arr[i].flops,
                                       "bytes": arr[i].bytes} for i in range(n.value)}

    def debug_poison_grad(self, index, value):
        self._check(self.lib.gpt_debug_poison_grad(self.h, index, value))

    def debug_wait_timeout(self, timeout_us) -> int:
        self._sync_stream()
        return self.lib.gpt_debug_wait_timeout(self.h, timeout_us)

    def train_step(self, tokens, targets, seg_ids, hp: AdamWConfig, loss=None, grad_norm=None, skipped=None):
        """forward_loss + backward + clip_adamw_step on the current stream, as
        one replayed CUDA graph (gpt_train_step)."""
        B, T = tokens.shape
        self._sync_stream()
        a = gpt_adamw(lr=hp.lr, beta1=hp.beta1, beta2=hp.beta2, eps=hp.eps, weight_decay=hp.weight_decay,
                      clip_norm=hp.clip_norm)
        return self._check(self.lib.gpt_train_step(self.h, _ptr(tokens), _ptr(targets), _ptr(seg_ids), B, T,
                                                   ctypes.byref(a), _ptr(loss), _ptr(grad_norm), _ptr(skipped)))
