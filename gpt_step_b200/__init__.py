"""Python binding of libgpt2step (the GPT-2 training step on one B200).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels. torch is used for device memory (the arena, token buffers) and for
the current CUDA stream. Importing this package does not load the library;
the first call that needs it does, and raises if it is missing.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgpt2step.so")

GPT2_PARAMS, GPT2_GRADS, GPT2_ADAM_M, GPT2_ADAM_V, GPT2_WEIGHTS_BF16 = 0, 1, 2, 3, 4
STATUS = {0: "GPT2_OK", 1: "GPT2_ERR_ARG", 2: "GPT2_ERR_CUDA", 3: "GPT2_ERR_TOKEN_RANGE",
          4: "GPT2_ERR_NONFINITE", 5: "GPT2_ERR_STATE", 6: "GPT2_ERR_TIMEOUT"}


class GPT2Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({_status_string(status)})")


class Config(ctypes.Structure):
    _fields_ = [("n_layer", ctypes.c_int32), ("n_head", ctypes.c_int32),
                ("n_embd", ctypes.c_int32), ("seq_len", ctypes.c_int32),
                ("vocab_real", ctypes.c_int32), ("vocab_padded", ctypes.c_int32),
                ("micro_batch", ctypes.c_int32), ("grad_accum", ctypes.c_int32),
                ("max_lr", ctypes.c_float), ("min_lr", ctypes.c_float),
                ("warmup_steps", ctypes.c_int32), ("total_steps", ctypes.c_int32),
                ("beta1", ctypes.c_float), ("beta2", ctypes.c_float), ("eps", ctypes.c_float),
                ("weight_decay", ctypes.c_float), ("grad_clip", ctypes.c_float)]

    @classmethod
    def make(cls, n_layer, n_head, n_embd, seq_len, vocab_real, vocab_padded=0, micro_batch=1,
             grad_accum=1, max_lr=6e-4, min_lr=0.0, warmup_steps=700, total_steps=18865,
             beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, grad_clip=1.0, **_):
        return cls(n_layer, n_head, n_embd, seq_len, vocab_real, vocab_padded, micro_batch,
                   grad_accum, max_lr, min_lr, warmup_steps, total_steps, beta1, beta2, eps,
                   weight_decay, grad_clip)


_lib_handle = None
_c = ctypes
_P = ctypes.c_void_p
_I = ctypes.c_int
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_F = ctypes.c_float
_FP = ctypes.POINTER(ctypes.c_float)
_SZ = ctypes.c_size_t

_SIGNATURES = {
    "gpt2_arena_bytes": (_SZ, [ctypes.POINTER(Config)]),
    "gpt2_num_params": (_I64, [ctypes.POINTER(Config), _I]),
    "gpt2_create": (_I, [ctypes.POINTER(Config), ctypes.c_uint64, _P, _SZ, _P, ctypes.POINTER(_P)]),
    "gpt2_destroy": (None, [_P]),
    "gpt2_fwd_bwd": (_I, [_P, _P, _P, _FP]),
    "gpt2_clip_adamw": (_I, [_P, _I32, _FP]),
    "gpt2_last_step_stats": (_I, [_P, _FP, _FP]),
    "gpt2_eval_loss": (_I, [_P, _P, _P, _I32, _FP]),
    "gpt2_train_step_host": (_I, [_P, _P, _P, _I32, _I32, _FP, _FP]),
    "gpt2_token_losses": (_I, [_P, _FP, _I64]),
    "gpt2_lr": (_F, [_P, _I32]),
    "gpt2_schedule_lr": (ctypes.c_double, [ctypes.POINTER(Config), _I32]),
    "gpt2_kernel_launches": (_I64, [_P]),
    "gpt2_profile_enable": (_I, [_P, _I]),
    "gpt2_profile_num_classes": (_I, []),
    "gpt2_profile_class_name": (ctypes.c_char_p, [_I]),
    "gpt2_profile_read": (_I, [_P, _I, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_I64),
                               ctypes.POINTER(ctypes.c_double)]),
    "gpt2_status_string": (ctypes.c_char_p, [_I]),
    "gpt2_num_tensors": (_I, [_P]),
    "gpt2_tensor_info": (_I, [_P, _I, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(_I64),
                              ctypes.POINTER(_I)]),
    "gpt2_read": (_I, [_P, _I, _I, _FP]),
    "gpt2_write": (_I, [_P, _I, _I, _FP]),
    "gpt2_state_device_ptr": (_I, [_P, _I, ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(_I64)]),
    "gpt2_num_buckets": (_I, [_P]),
    "gpt2_bucket_range": (_I, [_P, _I, ctypes.POINTER(_I64), ctypes.POINTER(_I64)]),
    "gpt2_set_bucket_events": (_I, [_P, ctypes.POINTER(_P), _I]),
    "gpt2_grad_sumsq": (_I, [_P, ctypes.POINTER(_I64), _I, _P]),
    "gpt2_clip_adamw_ranges": (_I, [_P, _I32, ctypes.POINTER(_I64), _I, _P, _FP]),
    "gpt2op_linear_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P, _P]),
    "gpt2op_linear_fwd_gelu": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P, _P]),
    "gpt2op_linear_dgrad": (_I, [_P, _P, _P, _P, _I, _I, _I, _P, _P]),
    "gpt2op_linear_wgrad": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P]),
    "gpt2op_linear_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, ctypes.POINTER(_I), _P, _P]),
    "gpt2op_bias_grad_workspace": (_SZ, [_I, _I]),
    "gpt2op_bias_grad": (_I, [_P, _P, _I, _I, _P, _SZ, _P]),
    "gpt2op_layernorm_fwd": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _P]),
    "gpt2op_layernorm_bwd_workspace": (_SZ, [_I, _I]),
    "gpt2op_layernorm_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _P, _SZ, _P]),
    "gpt2op_layernorm_bwd_noalloc_max_bytes": (_SZ, []),
    "gpt2op_layernorm_bwd_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _P]),
    "gpt2op_attention_fwd": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P]),
    "gpt2op_attention_bwd_workspace": (_SZ, [_I, _I, _I, _I]),
    "gpt2op_attention_bwd": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _SZ, _P, _P]),
    "gpt2op_softmax_ce": (_I, [_P, _P, _P, _I, _I, _I, _F, _P, _P]),
    "gpt2op_softmax_ce_masked": (_I, [_P, _P, _P, _I, _I, _I, _I, _F, _P, _P]),
    "gpt2op_lm_head_loss": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _P, _SZ, _P, _P]),
    "gpt2op_lm_head_ce_workspace": (_SZ, [_I, _I]),
    "gpt2op_lm_head_ce": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P, _SZ, _P, _P]),
    "gpt2op_embedding_fwd": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _P, _P]),
    "gpt2op_embedding_bwd": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "gpt2op_wait_selftest": (_I, [_I64, _P, _P]),
}


def lib():
    """Load libgpt2step.so (raises if it has not been built)."""
    global _lib_handle
    if _lib_handle is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m gpt_step_b200.build` (there is no fallback path)")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            f = getattr(h, name)
            f.restype = res
            f.argtypes = args
        _lib_handle = h
    return _lib_handle


def _status_string(st: int) -> str:
    try:
        return lib().gpt2_status_string(st).decode()
    except Exception:  # pragma: no cover
        return "?"


def check(st: int, what: str):
    if st != 0:
        raise GPT2Error(st, what)


def _ptr(t):
    """Device (or host numpy) pointer of a tensor/array, None for None."""
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _stream_handle(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def arena_bytes(cfg: Config) -> int:
    return lib().gpt2_arena_bytes(ctypes.byref(cfg))


def schedule_lr(cfg: Config, step: int) -> float:
    """The learning-rate schedule of `cfg` at `step` (host arithmetic in the library)."""
    return lib().gpt2_schedule_lr(ctypes.byref(cfg), step)


def num_params(cfg: Config, padded: bool = False) -> int:
    return lib().gpt2_num_params(ctypes.byref(cfg), 1 if padded else 0)


@dataclass
class TensorInfo:
    name: str
    shape: tuple


class GPT2:
    """One model: create(config, seed), fwd_bwd, clip_adamw, eval_loss, introspection."""

    def __init__(self, cfg: Config, seed: int, stream=None):
        import torch
        self.cfg = cfg
        self.torch = torch
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        nbytes = arena_bytes(cfg)
        if nbytes == 0:
            raise GPT2Error(1, "gpt2_arena_bytes (unsupported configuration)")
        self.arena = torch.empty(nbytes + 1024, dtype=torch.uint8, device="cuda")
        base = self.arena.data_ptr()
        self._base = (base + 1023) // 1024 * 1024
        h = ctypes.c_void_p()
        check(lib().gpt2_create(ctypes.byref(cfg), ctypes.c_uint64(seed), ctypes.c_void_p(self._base),
                                nbytes, ctypes.c_void_p(self.stream.cuda_stream), ctypes.byref(h)),
              "gpt2_create")
        self.h = h
        self.T = cfg.seq_len
        self.B = cfg.micro_batch
        self._infos = None

    def close(self):
        if getattr(self, "h", None):
            lib().gpt2_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- the step --------------------------------------------------------------------------
    def fwd_bwd(self, tokens, targets, want_loss: bool = False):
        out = ctypes.c_float()
        check(lib().gpt2_fwd_bwd(self.h, _ptr(tokens), _ptr(targets),
                                 ctypes.byref(out) if want_loss else None), "gpt2_fwd_bwd")
        return out.value if want_loss else None

    def clip_adamw(self, step: int, want_norm: bool = False):
        out = ctypes.c_float()
        check(lib().gpt2_clip_adamw(self.h, step, ctypes.byref(out) if want_norm else None),
              "gpt2_clip_adamw")
        return out.value if want_norm else None

    def last_step_stats(self):
        l, n = ctypes.c_float(), ctypes.c_float()
        check(lib().gpt2_last_step_stats(self.h, ctypes.byref(l), ctypes.byref(n)), "gpt2_last_step_stats")
        return l.value, n.value

    def eval_loss(self, tokens, targets) -> float:
        out = ctypes.c_float()
        check(lib().gpt2_eval_loss(self.h, _ptr(tokens), _ptr(targets), tokens.shape[0], ctypes.byref(out)),
              "gpt2_eval_loss")
        return out.value

    def train_step_host(self, tokens_host: np.ndarray, targets_host: np.ndarray, step: int):
        """tokens/targets: host int32 [n_micro, B, T] (pinned or pageable)."""
        l, n = ctypes.c_float(), ctypes.c_float()
        check(lib().gpt2_train_step_host(self.h, _ptr(tokens_host), _ptr(targets_host),
                                         tokens_host.shape[0], step, ctypes.byref(l), ctypes.byref(n)),
              "gpt2_train_step_host")
        return l.value, n.value

    def train_step_host_ptr(self, tok_ptr: int, tgt_ptr: int, n_micro: int, step: int):
        l, n = ctypes.c_float(), ctypes.c_float()
        check(lib().gpt2_train_step_host(self.h, tok_ptr, tgt_ptr, n_micro, step, ctypes.byref(l),
                                         ctypes.byref(n)), "gpt2_train_step_host")
        return l.value, n.value

    def token_losses(self) -> np.ndarray:
        out = np.empty(self.B * self.T, np.float32)
        check(lib().gpt2_token_losses(self.h, out.ctypes.data_as(_FP), out.size), "gpt2_token_losses")
        return out.reshape(self.B, self.T)

    def lr(self, step: int) -> float:
        return lib().gpt2_lr(self.h, step)

    def kernel_launches(self) -> int:
        return lib().gpt2_kernel_launches(self.h)

    def profile(self, on: bool):
        check(lib().gpt2_profile_enable(self.h, 1 if on else 0), "gpt2_profile_enable")

    def profile_read(self) -> dict:
        out = {}
        for c in range(lib().gpt2_profile_num_classes()):
            ms, n, work = ctypes.c_double(), ctypes.c_int64(), ctypes.c_double()
            check(lib().gpt2_profile_read(self.h, c, ctypes.byref(ms), ctypes.byref(n), ctypes.byref(work)),
                  "gpt2_profile_read")
            name = lib().gpt2_profile_class_name(c).decode()
            key = "flops" if name.startswith(("gemm", "attention")) else "bytes"
            out[name] = {"ms": ms.value, "launches": n.value, key: work.value}
        return out

    # -- introspection ---------------------------------------------------------------------
    def tensors(self):
        if self._infos is None:
            n = lib().gpt2_num_tensors(self.h)
            infos = []
            for i in range(n):
                name = ctypes.c_char_p()
                shape = (ctypes.c_int64 * 2)()
                nd = ctypes.c_int()
                check(lib().gpt2_tensor_info(self.h, i, ctypes.byref(name), shape, ctypes.byref(nd)),
                      "gpt2_tensor_info")
                infos.append(TensorInfo(name.value.decode(), tuple(shape[: nd.value])))
            self._infos = infos
        return self._infos

    def read(self, what: int, idx: int) -> np.ndarray:
        info = self.tensors()[idx]
        out = np.empty(info.shape, np.float32)
        check(lib().gpt2_read(self.h, what, idx, out.ctypes.data_as(_FP)), "gpt2_read")
        return out

    def write(self, what: int, idx: int, arr: np.ndarray):
        info = self.tensors()[idx]
        a = np.ascontiguousarray(arr, dtype=np.float32)
        if a.shape != info.shape:
            raise ValueError(f"{info.name}: shape {a.shape} != {info.shape}")
        check(lib().gpt2_write(self.h, what, idx, a.ctypes.data_as(_FP)), "gpt2_write")

    def state_tensor(self, what: int):
        """The flat state array `what` (fp32; bf16 for GPT2_WEIGHTS_BF16) as a torch view of the arena."""
        ptr, n = ctypes.c_void_p(), ctypes.c_int64()
        check(lib().gpt2_state_device_ptr(self.h, what, ctypes.byref(ptr), ctypes.byref(n)),
              "gpt2_state_device_ptr")
        off = ptr.value - self.arena.data_ptr()
        if what == GPT2_WEIGHTS_BF16:
            return self.arena[off: off + 2 * n.value].view(self.torch.bfloat16)
        return self.arena[off: off + 4 * n.value].view(self.torch.float32)

    # -- sharded optimizer step -------------------------------------------------------------
    def num_buckets(self) -> int:
        return lib().gpt2_num_buckets(self.h)

    def bucket_range(self, b: int):
        """(begin, end) elements of bucket b, or of the 1-D region for b = -1."""
        lo, hi = ctypes.c_int64(), ctypes.c_int64()
        check(lib().gpt2_bucket_range(self.h, b, ctypes.byref(lo), ctypes.byref(hi)), "gpt2_bucket_range")
        return lo.value, hi.value

    def set_bucket_events(self, events):
        """Register torch.cuda.Event objects (one per bucket); [] clears."""
        self._bucket_events = list(events)
        arr = (ctypes.c_void_p * max(1, len(events)))(*[e.cuda_event for e in events])
        check(lib().gpt2_set_bucket_events(self.h, arr, len(events)), "gpt2_set_bucket_events")

    @staticmethod
    def _ranges(ranges):
        flat = [int(v) for r in ranges for v in r]
        return (ctypes.c_int64 * len(flat))(*flat), len(ranges)

    def grad_sumsq(self, ranges, dev_out):
        """Enqueue: dev_out (a device float64 tensor of one element) = sum of g^2 over the ranges."""
        arr, n = self._ranges(ranges)
        check(lib().gpt2_grad_sumsq(self.h, arr, n, _ptr(dev_out)), "gpt2_grad_sumsq")

    def clip_adamw_ranges(self, step: int, ranges, dev_sumsq, want_norm: bool = False):
        arr, n = self._ranges(ranges)
        out = ctypes.c_float()
        check(lib().gpt2_clip_adamw_ranges(self.h, step, arr, n, _ptr(dev_sumsq),
                                           ctypes.byref(out) if want_norm else None), "gpt2_clip_adamw_ranges")
        return out.value if want_norm else None

    def read_all(self, what: int) -> dict:
        return {t.name: self.read(what, i) for i, t in enumerate(self.tensors())}

    def write_all(self, what: int, named: dict):
        for i, t in enumerate(self.tensors()):
            self.write(what, i, named[t.name])


# -- op-level calls (device tensors in, device tensors out) -----------------------------------

def _s(stream):
    return ctypes.c_void_p(_stream_handle(stream))


def linear_fwd(inp, w, bias, resid, out, err, stream=None):
    M, K = inp.shape
    N = w.shape[0]
    check(lib().gpt2op_linear_fwd(_ptr(inp), _ptr(w), _ptr(bias), _ptr(resid), _ptr(out), M, N, K,
                                  _ptr(err), _s(stream)), "gpt2op_linear_fwd")


def linear_fwd_gelu(inp, w, bias, pre_out, gelu_out, err, stream=None):
    M, K = inp.shape
    N = w.shape[0]
    check(lib().gpt2op_linear_fwd_gelu(_ptr(inp), _ptr(w), _ptr(bias), _ptr(pre_out), _ptr(gelu_out),
                                       M, N, K, _ptr(err), _s(stream)), "gpt2op_linear_fwd_gelu")


def linear_dgrad(dout, w, gelu_pre, din, err, stream=None):
    M, N = dout.shape
    K = w.shape[1]
    check(lib().gpt2op_linear_dgrad(_ptr(dout), _ptr(w), _ptr(gelu_pre), _ptr(din), M, N, K,
                                    _ptr(err), _s(stream)), "gpt2op_linear_dgrad")


def linear_wgrad(dout, inp, dw, err, splits=0, stream=None):
    M, N = dout.shape
    K = inp.shape[1]
    check(lib().gpt2op_linear_wgrad(_ptr(dout), _ptr(inp), _ptr(dw), M, N, K, splits, _ptr(err),
                                    _s(stream)), "gpt2op_linear_wgrad")


def linear_bwd(dout, w, inp, gelu_pre, din, dw, colsum, err, stream=None) -> int:
    """Grouped input + weight gradient of a linear layer; returns the dw reduction split."""
    M, N = dout.shape
    K = w.shape[1]
    sp = ctypes.c_int()
    check(lib().gpt2op_linear_bwd(_ptr(dout), _ptr(w), _ptr(inp), _ptr(gelu_pre), _ptr(din), _ptr(dw),
                                  _ptr(colsum), M, N, K, ctypes.byref(sp), _ptr(err), _s(stream)),
          "gpt2op_linear_bwd")
    return sp.value


def wait_selftest(limit_ns, err, stream=None) -> int:
    """Run the bounded-wait self-test; returns the raw status (6 = timed out as designed)."""
    return lib().gpt2op_wait_selftest(int(limit_ns), _ptr(err), _s(stream))


def bias_grad_workspace(M, N):
    return lib().gpt2op_bias_grad_workspace(M, N)


def bias_grad(dout, db, workspace, stream=None):
    M, N = dout.shape
    check(lib().gpt2op_bias_grad(_ptr(dout), _ptr(db), M, N, _ptr(workspace),
                                 0 if workspace is None else workspace.numel(), _s(stream)), "gpt2op_bias_grad")


def layernorm_fwd(x, w, b, y, mean, rstd, stream=None):
    rows, C = x.shape
    check(lib().gpt2op_layernorm_fwd(_ptr(x), _ptr(w), _ptr(b), _ptr(y), _ptr(mean), _ptr(rstd),
                                     rows, C, _s(stream)), "gpt2op_layernorm_fwd")


def layernorm_bwd_workspace(rows, C):
    return lib().gpt2op_layernorm_bwd_workspace(rows, C)


def layernorm_bwd(dy, x, mean, rstd, w, dresid, dx, dw, db, workspace, stream=None):
    rows, C = x.shape
    check(lib().gpt2op_layernorm_bwd(_ptr(dy), _ptr(x), _ptr(mean), _ptr(rstd), _ptr(w), _ptr(dresid),
                                     _ptr(dx), _ptr(dw), _ptr(db), rows, C, _ptr(workspace),
                                     0 if workspace is None else workspace.numel(), _s(stream)),
          "gpt2op_layernorm_bwd")


def layernorm_bwd_noalloc(dy, x, mean, rstd, w, dresid, dx, dw, db, stream=None):
    """LayerNorm backward with the library's own fixed scratch (no workspace argument)."""
    rows, C = x.shape
    check(lib().gpt2op_layernorm_bwd_noalloc(_ptr(dy), _ptr(x), _ptr(mean), _ptr(rstd), _ptr(w),
                                             _ptr(dresid), _ptr(dx), _ptr(dw), _ptr(db), rows, C,
                                             _s(stream)), "gpt2op_layernorm_bwd_noalloc")


def attention_fwd(qkv, out, lse, n_head, err, stream=None):
    B, T, C3 = qkv.shape
    hd = C3 // 3 // n_head
    check(lib().gpt2op_attention_fwd(_ptr(qkv), _ptr(out), _ptr(lse), B, T, n_head, hd, _ptr(err),
                                     _s(stream)), "gpt2op_attention_fwd")


def attention_bwd_workspace(B, T, H, hd):
    return lib().gpt2op_attention_bwd_workspace(B, T, H, hd)


def attention_bwd(qkv, out, dout, lse, dqkv, n_head, workspace, err, stream=None, dbias=None):
    """dbias (fp32 [3C]) or None: += the qkv bias gradient (column sums of dqkv)."""
    B, T, C3 = qkv.shape
    hd = C3 // 3 // n_head
    check(lib().gpt2op_attention_bwd(_ptr(qkv), _ptr(out), _ptr(dout), _ptr(lse), _ptr(dqkv), _ptr(dbias),
                                     B, T, n_head, hd, _ptr(workspace), workspace.numel(), _ptr(err),
                                     _s(stream)), "gpt2op_attention_bwd")


def softmax_ce(logits, targets, losses, V, dscale, err, stream=None):
    N, Vp = logits.shape
    check(lib().gpt2op_softmax_ce(_ptr(logits), _ptr(targets), _ptr(losses), N, V, Vp, dscale,
                                  _ptr(err), _s(stream)), "gpt2op_softmax_ce")


def softmax_ce_masked(logits, targets, losses, V, ignore_index, dscale, err, stream=None):
    """Softmax-CE where rows with target == ignore_index get loss 0 and zero gradient."""
    N, Vp = logits.shape
    check(lib().gpt2op_softmax_ce_masked(_ptr(logits), _ptr(targets), _ptr(losses), N, V, Vp, ignore_index,
                                         dscale, _ptr(err), _s(stream)), "gpt2op_softmax_ce_masked")


def lm_head_ce_workspace(N, Vp):
    return lib().gpt2op_lm_head_ce_workspace(N, Vp)


def lm_head_ce(h, wte, targets, logits, losses, V, dscale, write_grad, ws, err, stream=None):
    """Tied lm_head GEMM + softmax-CE: logits = h . wte^T, then losses (and dz in place)."""
    N, C = h.shape
    Vp = wte.shape[0]
    check(lib().gpt2op_lm_head_ce(_ptr(h), _ptr(wte), _ptr(targets), _ptr(logits), _ptr(losses), N, C, V, Vp,
                                  dscale, 1 if write_grad else 0, _ptr(ws),
                                  0 if ws is None else ws.numel() * ws.element_size(), _ptr(err), _s(stream)),
          "gpt2op_lm_head_ce")


def lm_head_loss(h, wte, targets, losses, V, ws, err, stream=None):
    """Per-row losses of the tied lm_head with the logits never stored."""
    N, C = h.shape
    Vp = wte.shape[0]
    check(lib().gpt2op_lm_head_loss(_ptr(h), _ptr(wte), _ptr(targets), _ptr(losses), N, C, V, Vp, _ptr(ws),
                                    0 if ws is None else ws.numel() * ws.element_size(), _ptr(err), _s(stream)),
          "gpt2op_lm_head_loss")


def embedding_fwd(tokens, wte, wpe, out, V, err, stream=None):
    B, T = tokens.shape
    C = wte.shape[1]
    check(lib().gpt2op_embedding_fwd(_ptr(tokens), _ptr(wte), _ptr(wpe), _ptr(out), B, T, C, V,
                                     _ptr(err), _s(stream)), "gpt2op_embedding_fwd")


def embedding_bwd(tokens, dx, dwte, dwpe, V, stream=None):
    B, T = tokens.shape
    C = dwte.shape[1]
    check(lib().gpt2op_embedding_bwd(_ptr(tokens), _ptr(dx), _ptr(dwte), _ptr(dwpe), B, T, C, V,
                                     _s(stream)), "gpt2op_embedding_bwd")
