"""B200-native forward pass + loss of the nanochat GPT block stack.

Thin ctypes binding of ``libnc.so`` (the C ABI declared in ``include/nc.h``).
This module only marshals arguments: every step of the forward runs in the
library's CUDA kernels.  PyTorch provides device memory and streams.  There is
no CPU fallback: if the library is missing or the device is not sm_100 every
call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

__all__ = [
    "NcError", "NcConfig", "lib", "init_config", "make_config", "check_config", "layer_window",
    "workspace_bytes", "forward_flops", "Model", "forward", "LaunchTrace", "KERNEL_KINDS", "get_status", "cast_bf16", "embedding",
    "rmsnorm", "rope_table", "rope_qknorm", "attention", "linear", "qkv_rope", "softcap_ce",
    "loss_mean", "cast_weights", "selftest_bounded_wait", "BF16", "F16", "F32",
    "fp8_quantize", "linear_fp8", "FP8_BLOCK", "FP8_LM_HEAD", "FP8_ALL",
    "train_workspace_bytes", "forward_backward", "linear_dgrad", "linear_wgrad", "attention_lse",
    "attention_backward",
    "EPI_STORE_16", "EPI_RELU2_16", "EPI_RESID_F32", "EPI_STORE_F32", "EPI_SOFTCAP_F32",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnc.so")

EPI_STORE_16, EPI_RELU2_16, EPI_RESID_F32, EPI_STORE_F32, EPI_SOFTCAP_F32 = range(5)
BF16, F16, F32 = 0, 1, 2  # nc_dtype (F32: fp8_quantize sources only)
DEV_TOKEN_RANGE, DEV_TARGET_RANGE, DEV_TIMEOUT, DEV_SMEM_ALIGN, DEV_POSITION = 0x1, 0x2, 0x4, 0x8, 0x10

STATUS_NAMES = {0: "NC_OK", 1: "NC_ERR_INVALID_ARG", 2: "NC_ERR_CONFIG", 3: "NC_ERR_SHAPE",
                4: "NC_ERR_ALIGNMENT", 5: "NC_ERR_WORKSPACE", 6: "NC_ERR_TOKEN_RANGE",
                7: "NC_ERR_TIMEOUT", 8: "NC_ERR_UNSUPPORTED_DEVICE", 9: "NC_ERR_CUDA", 10: "NC_ERR_F16_RANGE"}


class NcError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)}")


class NcConfig(ctypes.Structure):
    _fields_ = [("n_layer", ctypes.c_int32), ("d_model", ctypes.c_int32), ("n_head", ctypes.c_int32),
                ("n_kv_head", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("vocab", ctypes.c_int32),
                ("seq_len", ctypes.c_int32), ("short_window", ctypes.c_int32),
                ("window_pattern", ctypes.c_char * 8), ("softcap", ctypes.c_float),
                ("norm_eps", ctypes.c_float), ("rope_base", ctypes.c_float), ("act_dtype", ctypes.c_int32),
                ("extras", ctypes.c_uint32), ("fp8", ctypes.c_uint32)]

    def __repr__(self):
        return ("NcConfig(n_layer=%d, d_model=%d, n_head=%d, n_kv_head=%d, head_dim=%d, vocab=%d, "
                "seq_len=%d, short_window=%d, pattern=%r)" % (
                    self.n_layer, self.d_model, self.n_head, self.n_kv_head, self.head_dim,
                    self.vocab, self.seq_len, self.short_window, self.window_pattern.decode()))


_FPP = ctypes.POINTER(ctypes.c_void_p)


class NcWeights(ctypes.Structure):
    _fields_ = [("wte", ctypes.c_void_p), ("c_q", _FPP), ("c_k", _FPP), ("c_v", _FPP),
                ("attn_proj", _FPP), ("c_fc", _FPP), ("mlp_proj", _FPP), ("lm_head", ctypes.c_void_p),
                ("smear_gate", ctypes.c_void_p), ("value_embeds", _FPP), ("ve_gates", _FPP),
                ("resid_lambdas", ctypes.c_void_p), ("x0_lambdas", ctypes.c_void_p),
                ("backout_lambda", ctypes.c_void_p)]


class NcGrads(ctypes.Structure):
    _fields_ = [("wte", ctypes.c_void_p), ("c_q", _FPP), ("c_k", _FPP), ("c_v", _FPP),
                ("attn_proj", _FPP), ("c_fc", _FPP), ("mlp_proj", _FPP), ("lm_head", ctypes.c_void_p),
                ("smear_gate", ctypes.c_void_p), ("value_embeds", _FPP), ("ve_gates", _FPP),
                ("resid_lambdas", ctypes.c_void_p), ("x0_lambdas", ctypes.c_void_p),
                ("backout_lambda", ctypes.c_void_p)]


# Further terms of the full nanochat forward (bits of NcConfig.extras).
EXTRA_SMEAR, EXTRA_VALUE_EMBED, EXTRA_RESID_LAMBDAS, EXTRA_BACKOUT = 1, 2, 4, 8
EXTRA_ALL = 15

# Dynamic tensorwise e4m3 products (bits of NcConfig.fp8): the six block
# projections, the LM head.
FP8_BLOCK, FP8_LM_HEAD, FP8_ALL = 1, 2, 3


class NcTrace(ctypes.Structure):
    _fields_ = [("events", ctypes.POINTER(ctypes.c_void_p)), ("capacity", ctypes.c_int32),
                ("count", ctypes.c_int32), ("kinds", ctypes.POINTER(ctypes.c_int32))]


KERNEL_KINDS = ("rope_table", "cast", "embedding", "rmsnorm", "gemm_qkv", "rope_qknorm", "attention",
                "gemm_attn_proj", "gemm_fc", "gemm_mlp_proj", "gemm_lm_head", "ce_finalize", "loss_mean",
                "fp8_quant", "copy", "ce_bwd", "gemm_dgrad", "gemm_wgrad", "norm_bwd", "attn_bwd", "qk_bwd",
                "emb_bwd")

_lib = None


def lib():
    """The loaded CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m decoder_only_transformer_nc_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        cfgp = ctypes.POINTER(NcConfig)
        sigs = {
            "nc_init_config": (i32, [cfgp, i32, i32, i32, i32, i32, i32]),
            "nc_check_config": (i32, [cfgp]),
            "nc_layer_window": (i32, [cfgp, i32]),
            "nc_layer_value_embed": (i32, [cfgp, i32]),
            "nc_workspace_bytes": (sz, [cfgp, i32, i32]),
            "nc_forward_flops": (ctypes.c_double, [cfgp, i32, i32]),
            "nc_status_string": (ctypes.c_char_p, [i32]),
            "nc_version": (i32, []),
            "nc_forward": (i32, [cfgp, ctypes.POINTER(NcWeights), vp, vp, i32, i32, vp, vp, vp, vp, sz, vp]),
            "nc_forward_traced": (i32, [cfgp, ctypes.POINTER(NcWeights), vp, vp, i32, i32, vp, vp, vp, vp,
                                        sz, vp, ctypes.POINTER(NcTrace)]),
            "nc_event_create": (i32, [ctypes.POINTER(ctypes.c_void_p)]),
            "nc_event_destroy": (i32, [vp]),
            "nc_event_elapsed_ms": (i32, [vp, vp, ctypes.POINTER(ctypes.c_float)]),
            "nc_stream_wait_event": (i32, [vp, vp]),
            "nc_get_status": (i32, [vp, vp]),
            "nc_cast_weights": (i32, [vp, vp, i64, i32, vp]),
            "nc_embedding": (i32, [vp, vp, vp, i32, i32, i32, vp, vp]),
            "nc_rmsnorm": (i32, [vp, vp, i32, i32, f32, i32, vp]),
            "nc_rope_table": (i32, [vp, i32, i32, f32, vp]),
            "nc_rope_qknorm": (i32, [vp, vp, vp, i32, i32, i32, i32, i32, i64, i64, f32, i32, vp]),
            "nc_attention": (i32, [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp]),
            "nc_attention_strided": (i32, [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i64, i64, i32, vp]),
            "nc_linear": (i32, [vp, vp, vp, i32, i32, i32, i64, i32, f32, i32, vp, vp]),
            "nc_fp8_quantize": (i32, [vp, i32, i64, vp, vp, vp]),
            "nc_train_workspace_bytes": (sz, [cfgp, i32, i32]),
            "nc_forward_backward": (i32, [cfgp, ctypes.POINTER(NcWeights), vp, vp, i32, i32, vp,
                                          ctypes.POINTER(NcGrads), vp, sz, vp]),
            "nc_forward_backward_traced": (i32, [cfgp, ctypes.POINTER(NcWeights), vp, vp, i32, i32, vp,
                                                 ctypes.POINTER(NcGrads), vp, sz, vp, ctypes.POINTER(NcTrace)]),
            "nc_attention_lse": (i32, [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i64, i64, i32, vp]),
            "nc_attention_backward": (i32, [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp]),
            "nc_linear_dgrad": (i32, [vp, vp, vp, i32, i32, i32, i32, i32, vp, vp]),
            "nc_linear_wgrad": (i32, [vp, vp, vp, i32, i32, i32, f32, i32, vp, vp]),
            "nc_linear_fp8": (i32, [vp, vp, vp, vp, vp, i32, i32, i32, i64, i32, f32, i32, vp, vp]),
            "nc_qkv_rope": (i32, [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, i32, vp, vp]),
            "nc_softcap_ce": (i32, [vp, vp, vp, vp, i32, i32, f32, vp, vp]),
            "nc_loss_mean": (i32, [vp, vp, i32, i32, vp, vp]),
            "nc_selftest_bounded_wait": (i32, [vp, ctypes.c_uint32, vp]),
            "nc_session_bytes": (sz, [cfgp, i32, i32]),
            "nc_prefill_workspace_bytes": (sz, [cfgp, i32, i32]),
            "nc_prefill": (i32, [cfgp, ctypes.POINTER(NcWeights), vp, i32, i32, vp, vp, sz, i32, vp, sz, vp]),
            "nc_decode_step": (i32, [cfgp, ctypes.POINTER(NcWeights), vp, i32, i32, vp, vp, sz, i32, vp]),
            "nc_decode_step_dev": (i32, [cfgp, ctypes.POINTER(NcWeights), vp, i32, vp, vp, vp, sz, i32, vp]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(code: int, where: str):
    if code != 0:
        raise NcError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


# ---------------------------------------------------------------- configuration

def init_config(depth: int, aspect_ratio: int = 64, head_dim: int = 128, n_kv_head: int = 0,
                seq_len: int = 2048, vocab: int = 32768) -> NcConfig:
    c = NcConfig()
    _check(lib().nc_init_config(ctypes.byref(c), depth, aspect_ratio, head_dim, n_kv_head, seq_len,
                                vocab), "nc_init_config")
    return c


def make_config(n_layer, d_model, n_head, n_kv_head, head_dim, seq_len, vocab, short_window=0,
                window_pattern="SSSL", softcap=15.0, norm_eps=1e-6, rope_base=10000.0,
                act_dtype=F16, extras=0, fp8=0) -> NcConfig:
    c = NcConfig(n_layer, d_model, n_head, n_kv_head, head_dim, vocab, seq_len,
                 short_window if short_window > 0 else seq_len // 4, window_pattern.encode(),
                 softcap, norm_eps, rope_base, act_dtype, extras, fp8)
    _check(lib().nc_check_config(ctypes.byref(c)), "nc_check_config")
    return c


def check_config(c: NcConfig) -> int:
    return lib().nc_check_config(ctypes.byref(c))


def layer_window(c: NcConfig, layer: int) -> int:
    return lib().nc_layer_window(ctypes.byref(c), layer)


def layer_value_embed(c: NcConfig, layer: int) -> int:
    return lib().nc_layer_value_embed(ctypes.byref(c), layer)


def workspace_bytes(c: NcConfig, B: int, T: int) -> int:
    return lib().nc_workspace_bytes(ctypes.byref(c), B, T)


def forward_flops(c: NcConfig, B: int, T: int) -> float:
    return lib().nc_forward_flops(ctypes.byref(c), B, T)


# ---------------------------------------------------------------- model

@dataclass
class Model:
    """fp32 weights resident on the device plus the nc_weights view of them."""

    cfg: NcConfig
    tensors: dict
    weights: NcWeights
    _keep: list

    @classmethod
    def from_tensors(cls, cfg: NcConfig, t: dict) -> "Model":
        """t: {"wte", "lm_head", "layers": [{c_q, c_k, c_v, attn_proj, c_fc, mlp_proj}]}
        with contiguous float32 CUDA tensors in [out, in] layout, and optionally
        t["extras"] = {"smear_gate", "resid_lambdas", "x0_lambdas",
        "backout_lambda", "value_embeds": [L], "ve_gates": [L]} (list entries may
        be None) for the terms enabled in cfg.extras."""
        L = cfg.n_layer
        arrs = {}
        for name in ("c_q", "c_k", "c_v", "attn_proj", "c_fc", "mlp_proj"):
            a = (ctypes.c_void_p * L)(*[t["layers"][l][name].data_ptr() for l in range(L)])
            arrs[name] = a
        ex = t.get("extras") or {}
        p = lambda x: None if x is None else x.data_ptr()
        for name in ("value_embeds", "ve_gates"):
            lst = ex.get(name)
            arrs[name] = None if lst is None else (ctypes.c_void_p * L)(*[p(v) for v in lst])
        fpp = lambda a: None if a is None else ctypes.cast(a, _FPP)
        w = NcWeights(t["wte"].data_ptr(), *[ctypes.cast(arrs[n], _FPP) for n in
                                             ("c_q", "c_k", "c_v", "attn_proj", "c_fc", "mlp_proj")],
                      t["lm_head"].data_ptr(), p(ex.get("smear_gate")), fpp(arrs["value_embeds"]),
                      fpp(arrs["ve_gates"]), p(ex.get("resid_lambdas")), p(ex.get("x0_lambdas")),
                      p(ex.get("backout_lambda")))
        return cls(cfg, t, w, [a for a in arrs.values() if a is not None])

    @classmethod
    def from_numpy(cls, cfg: NcConfig, w: dict, device="cuda", extras: dict | None = None) -> "Model":
        """As from_tensors, from float32 numpy arrays.  ``extras`` holds the further
        weights (numpy, the layout of ``from_tensors``); only the tables of layers
        that use a value embedding are copied to the device."""
        import torch
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device).contiguous()
        t = {"wte": dev(w["wte"]), "lm_head": dev(w["lm_head"]),
             "layers": [{k: dev(v) for k, v in lw.items()} for lw in w["layers"]]}
        if extras:
            e = {}
            for k in ("smear_gate", "resid_lambdas", "x0_lambdas"):
                if extras.get(k) is not None:
                    e[k] = dev(extras[k])
            if extras.get("backout_lambda") is not None:
                e["backout_lambda"] = dev(np.asarray(extras["backout_lambda"], dtype=np.float32).reshape(1))
            if extras.get("value_embeds") is not None:
                use = [layer_value_embed(cfg, l) == 1 for l in range(cfg.n_layer)]
                e["value_embeds"] = [dev(v) if u and v is not None else None
                                     for u, v in zip(use, extras["value_embeds"])]
                e["ve_gates"] = [dev(g) if u and g is not None else None
                                 for u, g in zip(use, extras["ve_gates"])]
            t["extras"] = e
        return cls.from_tensors(cfg, t)


def forward(model: Model, tokens, targets=None, want_logits=False, want_token_loss=False,
            workspace=None, stream=None, out=None, trace: "LaunchTrace | None" = None):
    """Runs nc_forward.  tokens/targets: int32 CUDA tensors [B, T].

    Returns a dict of CUDA tensors: ``loss`` (scalar, if targets), ``token_loss``
    ([B,T], if asked), ``logits`` ([B,T,V] fp32 soft-capped, if asked) and the
    ``workspace`` used (its first word is the device status of the call).
    ``out`` may hold preallocated tensors under the same keys.
    """
    import torch
    cfg = model.cfg
    B, T = tokens.shape
    out = {} if out is None else out
    dev = tokens.device
    need = workspace_bytes(cfg, B, T)
    if need == 0:
        raise NcError(3, "nc_workspace_bytes")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    res = {"workspace": workspace}
    logits = tl = loss = None
    if want_logits:
        logits = out.get("logits")
        if logits is None:
            logits = torch.empty((B, T, cfg.vocab), dtype=torch.float32, device=dev)
        res["logits"] = logits
    if targets is not None:
        loss = out.get("loss")
        if loss is None:
            loss = torch.empty((), dtype=torch.float32, device=dev)
        res["loss"] = loss
        if want_token_loss:
            tl = out.get("token_loss")
            if tl is None:
                tl = torch.empty((B, T), dtype=torch.float32, device=dev)
            res["token_loss"] = tl
    _check(lib().nc_forward_traced(ctypes.byref(cfg), ctypes.byref(model.weights), _ptr(tokens),
                                   _ptr(targets), B, T, _ptr(logits), _ptr(tl), _ptr(loss),
                                   _ptr(workspace), workspace.numel(), _stream(stream),
                                   None if trace is None else ctypes.byref(trace.struct)),
           "nc_forward")
    return res


class Session:
    """KV-cache inference state on the device (see nc_prefill / nc_decode_step):
    the weights cast once, the RoPE table and every layer's cache for B rows of
    up to T_max positions."""

    def __init__(self, model: Model, B: int, T_max: int, device="cuda"):
        import torch
        n = lib().nc_session_bytes(ctypes.byref(model.cfg), B, T_max)
        if n == 0:
            raise NcError(3, "nc_session_bytes")
        self.model, self.B, self.T_max = model, B, T_max
        self.buffer = torch.empty(n, dtype=torch.uint8, device=device)
        self.pos = 0
        self._graph = None

    def prefill(self, tokens, want_logits=False, stream=None):
        """Runs the prompt tokens [B, T]; returns the logits [B, T, V] if asked."""
        import torch
        cfg = self.model.cfg
        B, T = tokens.shape
        ws = torch.empty(max(1, lib().nc_prefill_workspace_bytes(ctypes.byref(cfg), B, T)), dtype=torch.uint8,
                         device=tokens.device)
        logits = torch.empty((B, T, cfg.vocab), dtype=torch.float32, device=tokens.device) if want_logits else None
        _check(lib().nc_prefill(ctypes.byref(cfg), ctypes.byref(self.model.weights), _ptr(tokens), B, T,
                                _ptr(logits), _ptr(self.buffer), self.buffer.numel(), self.T_max, _ptr(ws),
                                ws.numel(), _stream(stream)), "nc_prefill")
        self.pos = T
        return logits

    def decode(self, tokens, logits=None, stream=None):
        """One position for every row: tokens [B] int32; returns logits [B, V]."""
        import torch
        cfg = self.model.cfg
        if logits is None:
            logits = torch.empty((self.B, cfg.vocab), dtype=torch.float32, device=tokens.device)
        _check(lib().nc_decode_step(ctypes.byref(cfg), ctypes.byref(self.model.weights), _ptr(tokens), self.B,
                                    self.pos, _ptr(logits), _ptr(self.buffer), self.buffer.numel(), self.T_max,
                                    _stream(stream)), "nc_decode_step")
        self.pos += 1
        return logits

    def _step_dev(self, stream=None):
        cfg = self.model.cfg
        _check(lib().nc_decode_step_dev(ctypes.byref(cfg), ctypes.byref(self.model.weights), _ptr(self._g_tokens),
                                        self.B, _ptr(self._g_pos), _ptr(self._g_logits), _ptr(self.buffer),
                                        self.buffer.numel(), self.T_max, _stream(stream)), "nc_decode_step_dev")

    def decode_graph(self, tokens):
        """As ``decode``, through one CUDA graph of the step replayed for every
        further position (the position lives in device memory,
        nc_decode_step_dev).  tokens [B] int32 are copied into the graph's input;
        the returned logits [B, V] are the graph's buffer, overwritten by the
        next step.  The first call runs the step eagerly, then captures it.
        Raises NcError(NC_ERR_SHAPE) once every cache position is used."""
        import torch
        if self.pos >= self.T_max:
            raise NcError(3, f"Session.decode_graph: position {self.pos} is past the cache (T_max {self.T_max})")
        if self._graph is None:
            cfg = self.model.cfg
            dev = tokens.device
            self._g_tokens = tokens.clone()
            self._g_logits = torch.empty((self.B, cfg.vocab), dtype=torch.float32, device=dev)
            self._g_pos = torch.full((4,), self.pos, dtype=torch.int32, device=dev)
            self._step_dev()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self._step_dev()
            self._graph = g
        else:
            self._g_tokens.copy_(tokens)
            self._graph.replay()
        self.pos += 1
        return self._g_logits

    def status(self):
        return get_status(self.buffer)


class LaunchTrace:
    """Per-launch CUDA events for one traced forward (see nc_forward_traced)."""

    def __init__(self, capacity: int):
        L = lib()
        self.capacity = capacity
        self._ev = (ctypes.c_void_p * (2 * capacity))()
        for i in range(2 * capacity):
            h = ctypes.c_void_p()
            _check(L.nc_event_create(ctypes.byref(h)), "nc_event_create")
            self._ev[i] = h
        self._kinds = (ctypes.c_int32 * capacity)()
        self.struct = NcTrace(ctypes.cast(self._ev, ctypes.POINTER(ctypes.c_void_p)), capacity, 0,
                              ctypes.cast(self._kinds, ctypes.POINTER(ctypes.c_int32)))

    def launches(self):
        """[(kind name, milliseconds)] of the last traced forward (waits for it)."""
        L = lib()
        out = []
        ms = ctypes.c_float()
        for i in range(self.struct.count):
            _check(L.nc_event_elapsed_ms(self._ev[2 * i], self._ev[2 * i + 1], ctypes.byref(ms)),
                   "nc_event_elapsed_ms")
            out.append((KERNEL_KINDS[self._kinds[i]], ms.value))
        return out

    def kinds(self):
        """Kind names of the last traced call's launches (known once it is enqueued)."""
        return [KERNEL_KINDS[self._kinds[i]] for i in range(self.struct.count)]

    def end_event(self, i: int):
        """The event recorded right after launch i (a cudaEvent_t handle)."""
        if not 0 <= i < self.struct.count:
            raise IndexError(f"launch {i} of {self.struct.count}")
        return self._ev[2 * i + 1]

    def close(self):
        if self._ev is not None:
            for i in range(2 * self.capacity):
                lib().nc_event_destroy(self._ev[i])
            self._ev = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def get_status(status_tensor, stream=None) -> int:
    """Synchronises the stream and returns the nc_status of a device status word."""
    return lib().nc_get_status(_ptr(status_tensor), _stream(stream))


# ---------------------------------------------------------------- single steps

def _dt(t):
    """nc_dtype of a 16-bit torch tensor."""
    import torch
    if t.dtype == torch.float16:
        return F16
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"expected a float16 or bfloat16 tensor, got {t.dtype}")


def cast_weights(src, dst, stream=None):
    """fp32 -> bf16-rounded weights in dst's format (bfloat16, or float16 holding the bf16 values)."""
    _check(lib().nc_cast_weights(_ptr(src), _ptr(dst), src.numel(), _dt(dst), _stream(stream)),
           "nc_cast_weights")


def embedding(tokens, wte, x, status=None, stream=None):
    M = tokens.numel()
    V, C = wte.shape
    _check(lib().nc_embedding(_ptr(tokens), _ptr(wte), _ptr(x), M, C, V, _ptr(status), _stream(stream)),
           "nc_embedding")


def rmsnorm(x, out, eps=1e-6, stream=None):
    C = x.shape[-1]
    _check(lib().nc_rmsnorm(_ptr(x), _ptr(out), x.numel() // C, C, eps, _dt(out), _stream(stream)),
           "nc_rmsnorm")


def rope_table(table, T, D, base=10000.0, stream=None):
    _check(lib().nc_rope_table(_ptr(table), T, D, base, _stream(stream)), "nc_rope_table")


def rope_qknorm(q, k, table, B, T, H, Hkv, D, q_row_stride=None, k_row_stride=None, eps=1e-6,
                stream=None):
    qs = H * D if q_row_stride is None else q_row_stride
    ks = Hkv * D if k_row_stride is None else k_row_stride
    _check(lib().nc_rope_qknorm(_ptr(q), _ptr(k), _ptr(table), B, T, H, Hkv, D, qs, ks, eps, _dt(q),
                                _stream(stream)), "nc_rope_qknorm")


def attention(q, k, v, out, window, stream=None):
    B, T, H, D = q.shape
    Hkv = k.shape[2]
    _check(lib().nc_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, T, H, Hkv, D, window, _dt(q),
                              _stream(stream)), "nc_attention")


def linear(a, w, out, epilogue, cap=15.0, status=None, stream=None):
    M, K = a.shape
    N = w.shape[0]
    _check(lib().nc_linear(_ptr(a), _ptr(w), _ptr(out), M, N, K, out.stride(0), epilogue, cap, _dt(a),
                           _ptr(status), _stream(stream)), "nc_linear")


def fp8_quantize(x, codes, amax, stream=None):
    """Dynamic tensorwise e4m3 codes of x (fp32, bf16 or fp16 device tensor)
    into codes (uint8, same element count); amax: one-element fp32 tensor."""
    import torch
    dt = {torch.float32: F32, torch.bfloat16: BF16, torch.float16: F16}[x.dtype]
    _check(lib().nc_fp8_quantize(_ptr(x), dt, x.numel(), _ptr(codes), _ptr(amax), _stream(stream)),
           "nc_fp8_quantize")


def linear_fp8(a8, amax_a, w8, amax_w, out, epilogue, cap=15.0, dtype=F16, status=None, stream=None):
    """out = epilogue((a8 @ w8^T) / (s_a s_w)) on e4m3 codes (uint8 tensors)."""
    M, K = a8.shape
    N = w8.shape[0]
    _check(lib().nc_linear_fp8(_ptr(a8), _ptr(amax_a), _ptr(w8), _ptr(amax_w), _ptr(out), M, N, K,
                               out.stride(0), epilogue, cap, dtype, _ptr(status), _stream(stream)),
           "nc_linear_fp8")


def train_workspace_bytes(c: NcConfig, B: int, T: int) -> int:
    return lib().nc_train_workspace_bytes(ctypes.byref(c), B, T)


def forward_backward(model: Model, tokens, targets, grads: dict | None = None, workspace=None, stream=None,
                     loss=None, trace: "LaunchTrace | None" = None):
    """The training micro-step's forward + loss.backward() (nc_forward_backward).

    tokens/targets: int32 CUDA tensors [B, T].  ``grads`` (optional) holds fp32
    CUDA tensors in the layout of ``Model.tensors`` ("wte", "lm_head",
    "layers": [{c_q, ...}], and "extras" with the same keys as the model's for
    the terms enabled in cfg.extras); the gradients are ADDED to them.  Without
    it, zeroed tensors are made.  Returns (loss: scalar CUDA tensor, grads,
    workspace).
    """
    import torch
    cfg = model.cfg
    B, T = tokens.shape
    need = train_workspace_bytes(cfg, B, T)
    if need == 0:
        raise NcError(2, "nc_train_workspace_bytes")
    dev = tokens.device
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    t = model.tensors
    if grads is None:
        z = lambda x: None if x is None else torch.zeros_like(x)
        grads = {"wte": z(t["wte"]), "lm_head": z(t["lm_head"]),
                 "layers": [{k: z(lw[k]) for k in ("c_q", "c_k", "c_v", "attn_proj", "c_fc", "mlp_proj")}
                            for lw in t["layers"]]}
        tex = t.get("extras") or {}
        if tex:
            grads["extras"] = {k: ([z(x) for x in v] if isinstance(v, list) else z(v)) for k, v in tex.items()}
    L = cfg.n_layer
    arrs = [(ctypes.c_void_p * L)(*[grads["layers"][l][n].data_ptr() for l in range(L)])
            for n in ("c_q", "c_k", "c_v", "attn_proj", "c_fc", "mlp_proj")]
    gex = grads.get("extras") or {}
    p = lambda x: None if x is None else x.data_ptr()
    per_layer = {}
    for name in ("value_embeds", "ve_gates"):
        lst = gex.get(name)
        per_layer[name] = None if lst is None else (ctypes.c_void_p * L)(*[p(x) for x in lst])
    fpp = lambda a: None if a is None else ctypes.cast(a, _FPP)
    g = NcGrads(grads["wte"].data_ptr(), *[ctypes.cast(a, _FPP) for a in arrs], grads["lm_head"].data_ptr(),
                p(gex.get("smear_gate")), fpp(per_layer["value_embeds"]), fpp(per_layer["ve_gates"]),
                p(gex.get("resid_lambdas")), p(gex.get("x0_lambdas")), p(gex.get("backout_lambda")))
    if loss is None:
        loss = torch.empty((), dtype=torch.float32, device=dev)
    _check(lib().nc_forward_backward_traced(ctypes.byref(cfg), ctypes.byref(model.weights), _ptr(tokens),
                                            _ptr(targets), B, T, _ptr(loss), ctypes.byref(g), _ptr(workspace),
                                            workspace.numel(), _stream(stream),
                                            None if trace is None else ctypes.byref(trace.struct)),
           "nc_forward_backward")
    return loss, grads, workspace


def attention_lse(qkv, out, lse, H, Hkv, D, window, stream=None):
    """Forward attention on a packed qkv [B, T, (H + 2 Hkv) D] tensor; out [B, T, H*D], lse [B, T, H] fp32."""
    B, T, W = qkv.shape
    q = qkv.view(B * T, W)
    _check(lib().nc_attention_lse(_ptr(q), ctypes.c_void_p(q.data_ptr() + H * D * q.element_size()),
                                  ctypes.c_void_p(q.data_ptr() + (H + Hkv) * D * q.element_size()), _ptr(out),
                                  _ptr(lse), B, T, H, Hkv, D, window, W, W, _dt(qkv), _stream(stream)),
           "nc_attention_lse")


def attention_backward(qkv, o, dO, lse, dqkv, H, Hkv, D, window, delta=None, stream=None):
    """dq | dk | dv into dqkv (qkv's packed layout) from o, dO and lse."""
    import torch
    B, T, _ = qkv.shape
    if delta is None:
        delta = torch.empty((B, T, H), dtype=torch.float32, device=qkv.device)
    _check(lib().nc_attention_backward(_ptr(qkv), _ptr(o), _ptr(dO), _ptr(lse), _ptr(delta), _ptr(dqkv), B, T, H,
                                       Hkv, D, window, _dt(qkv), _stream(stream)), "nc_attention_backward")


def linear_dgrad(dy, w, dx, status=None, stream=None):
    """dx [M, K] = dy [M, N] . w [N, K]; dx fp32 or 16-bit (same format as dy)."""
    import torch
    M, N = dy.shape
    K = w.shape[1]
    epi = EPI_STORE_F32 if dx.dtype == torch.float32 else EPI_STORE_16
    _check(lib().nc_linear_dgrad(_ptr(dy), _ptr(w), _ptr(dx), M, N, K, epi, _dt(dy), _ptr(status),
                                 _stream(stream)), "nc_linear_dgrad")


def linear_wgrad(dy, x, dw, alpha=1.0, status=None, stream=None):
    """dw [N, K] += alpha dy [M, N]^T . x [M, K] (fp32)."""
    M, N = dy.shape
    K = x.shape[1]
    _check(lib().nc_linear_wgrad(_ptr(dy), _ptr(x), _ptr(dw), M, N, K, alpha, _dt(dy), _ptr(status),
                                 _stream(stream)), "nc_linear_wgrad")


def qkv_rope(a, w, out, table, T, H, Hkv, D, eps=1e-6, status=None, stream=None):
    M, C = a.shape
    _check(lib().nc_qkv_rope(_ptr(a), _ptr(w), _ptr(out), _ptr(table), M, T, C, H, Hkv, D, eps, _dt(a),
                             _ptr(status), _stream(stream)), "nc_qkv_rope")


def softcap_ce(z, targets, token_loss, capped_out=None, cap=15.0, status=None, stream=None):
    M, V = z.shape
    _check(lib().nc_softcap_ce(_ptr(z), _ptr(targets), _ptr(capped_out), _ptr(token_loss), M, V, cap,
                               _ptr(status), _stream(stream)), "nc_softcap_ce")


def selftest_bounded_wait(status, limit_us=20000, stream=None):
    _check(lib().nc_selftest_bounded_wait(_ptr(status), limit_us, _stream(stream)),
           "nc_selftest_bounded_wait")


def loss_mean(token_loss, targets, V, loss, stream=None):
    _check(lib().nc_loss_mean(_ptr(token_loss), _ptr(targets), token_loss.numel(), V, _ptr(loss),
                              _stream(stream)), "nc_loss_mean")
