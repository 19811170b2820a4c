"""ctypes binding of liborthrus (include/orthrus.h).

Argument marshalling only: every computation runs in the library's sm_100a
kernels. PyTorch provides device memory and the current CUDA stream. Loading
fails loudly when the library has not been built; there is no fallback.

The function names mirror the C entry points without the ``orthrus_`` prefix.
``DeviceModel`` owns the device buffers a plan needs (weights uploaded from
host arrays, the KV cache, the workspace) and the host plan buffer.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liborthrus.so")

KIND_NAMES = ["embed", "rmsnorm", "gemm_qkv", "attention", "gemm_o", "gemm_gate_up", "gemm_down", "lm_head",
              "argmax", "accept", "other", "end", "forward", "sample"]

OK, ERR_ARG, ERR_CAPACITY, ERR_CUDA, ERR_TIMEOUT, ERR_NAN, ERR_UNSUPPORTED, ERR_WORKSPACE = range(8)
STATUS_NAMES = {0: "OK", 1: "ARG", 2: "CAPACITY", 3: "CUDA", 4: "TIMEOUT", 5: "NAN", 6: "UNSUPPORTED",
                7: "WORKSPACE"}


class OrthrusError(RuntimeError):
    def __init__(self, call, code):
        super().__init__(f"{call} returned {STATUS_NAMES.get(code, code)}")
        self.code = code


class Config(C.Structure):
    _fields_ = [(n, C.c_int32) for n in ("n_layers", "d_model", "n_heads", "n_kv_heads", "head_dim", "d_ff",
                                          "vocab", "mask_id", "qk_norm")] + [("rope_theta", C.c_float),
                                                                             ("rms_eps", C.c_float)]


_PP = C.POINTER(C.c_void_p)


class Weights(C.Structure):
    _fields_ = [("embed", C.c_void_p), ("final_norm", C.c_void_p), ("lm_head", C.c_void_p)] + [
        (n, _PP) for n in ("attn_norm", "mlp_norm", "w_qkv", "w_o", "q_norm", "k_norm", "w_gate_up", "w_down",
                           "wd_qkv", "wd_o", "wd_q_norm", "wd_k_norm")]


class Cache(C.Structure):
    _fields_ = [("k", C.c_void_p), ("v", C.c_void_p), ("len", C.c_void_p), ("batch", C.c_int32),
                ("capacity", C.c_int32)]


class AcceptStats(C.Structure):
    _fields_ = [("accepted", C.c_float), ("rejected", C.c_float)]


# (name, restype, argtypes) for every symbol of include/orthrus.h
_I32, _SZ, _VP, _F = C.c_int32, C.c_size_t, C.c_void_p, C.c_float
_PCFG = C.POINTER(Config)
_PST = C.POINTER(AcceptStats)
SIGNATURES = [
    ("orthrus_plan_bytes", _SZ, [_PCFG]),
    ("orthrus_workspace_bytes", _SZ, [_PCFG, _I32, _I32, _I32, _I32]),
    ("orthrus_block_scratch_offset", _SZ, [_PCFG, _I32, _I32, _I32, _I32]),
    ("orthrus_block_scratch_bytes", _SZ, [_PCFG, _I32, _I32]),
    ("orthrus_plan_init", _I32, [_VP, _SZ, _PCFG, C.POINTER(Weights), C.POINTER(Cache), _I32, _I32, _VP, _SZ, _VP]),
    ("orthrus_status_ptr", _VP, [_VP]),
    ("orthrus_clear_status", _I32, [_VP, _VP]),
    ("orthrus_decode_step_launches", _I32, [_VP, _I32]),
    ("orthrus_trace", _I32, [_VP, _VP, _VP, _I32, _VP]),
    ("orthrus_timeline_bytes", _SZ, [_VP]),
    ("orthrus_timeline", _I32, [_VP, _VP, _SZ]),
    ("orthrus_prefill", _I32, [_VP, _VP, _VP, _I32, _VP, _VP]),
    ("orthrus_draft_block", _I32, [_VP, _VP, _I32, _VP, _VP, _VP]),
    ("orthrus_verify_block", _I32, [_VP, _VP, _VP, _I32, _VP, _VP, _VP]),
    ("orthrus_accept_commit", _I32, [_VP, _VP, _VP, _VP, _I32, _VP, _VP, _I32, _VP]),
    ("orthrus_decode_step", _I32, [_VP, _VP, _I32, _VP, _VP, _VP, _VP]),
    ("orthrus_draft_refine", _I32, [_VP, _VP, _VP, _I32, _VP, _VP, _VP]),
    ("orthrus_decode_step_ex", _I32, [_VP, _VP, _I32, _I32, _VP, _VP, _VP, _VP]),
    ("orthrus_sample_tokens", _I32, [_VP, _I32, _I32, _F, _VP, _VP, _VP, _VP]),
    ("orthrus_accept_sample", _I32, [_VP, _VP, _VP, _VP, _VP, _I32, _F, _VP, _VP, _VP, _VP, _VP]),
    ("orthrus_decode_step_sampled", _I32, [_VP, _VP, _I32, _F, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    ("orthrus_attention_workspace_bytes", _SZ, [_I32, _I32, _I32, _I32, _I32, _I32]),
    ("orthrus_attention", _I32, [_VP, _VP, _VP, _VP, _VP, _VP, _I32, _I32, _I32, _I32, _I32, _I32, _I32, _I32, _VP,
                                 _VP, _SZ, _VP, _VP]),
    ("orthrus_linear_workspace_bytes", _SZ, [_I32, _I32, _I32]),
    ("orthrus_linear", _I32, [_VP, _VP, _VP, _I32, _I32, _I32, _VP, _SZ, _VP, _VP]),
    ("orthrus_linear_noalloc", _I32, [_VP, _VP, _VP, _I32, _I32, _I32, _VP, _VP]),
    ("orthrus_accept_stats_update", _I32, [_PST, _VP, _I32, _I32, _F]),
    ("orthrus_accept_rate", _F, [_PST]),
    ("orthrus_choose_block_size", _I32, [_PST, _I32, _VP, _VP, _I32]),
]

_lib = None


def load(path: str = LIB_PATH):
    """Load liborthrus.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise FileNotFoundError(f"{path} is missing: build it with `python -m shared_kv_draft_b200.build`")
        lib = C.CDLL(path)
        for name, res, args in SIGNATURES:
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _check(name, code):
    if code != OK:
        raise OrthrusError(name, code)


def make_config(shape) -> Config:
    return Config(shape.n_layers, shape.d_model, shape.n_heads, shape.n_kv_heads, shape.head_dim, shape.d_ff,
                  shape.vocab, shape.mask_id, int(bool(shape.qk_norm)), float(shape.rope_theta), float(shape.rms_eps))


# ---- thin wrappers with the C names -----------------------------------------------------------

def plan_bytes(cfg: Config) -> int:
    return load().orthrus_plan_bytes(C.byref(cfg))


def workspace_bytes(cfg: Config, batch: int, capacity: int, max_block: int, max_rows: int) -> int:
    return load().orthrus_workspace_bytes(C.byref(cfg), batch, capacity, max_block, max_rows)


def block_scratch_bytes(cfg: Config, batch: int, max_block: int) -> int:
    return load().orthrus_block_scratch_bytes(C.byref(cfg), batch, max_block)


def block_scratch_offset(cfg: Config, batch: int, capacity: int, max_block: int, max_rows: int) -> int:
    return load().orthrus_block_scratch_offset(C.byref(cfg), batch, capacity, max_block, max_rows)


def attention(q, k_cache, v_cache, k_blk, v_blk, lens, batch, n_kv_heads, group, Q, head_dim, capacity, blk_stride,
              mode, out, workspace, status, stream=None):
    """q, K and V in fp16 (device); out: bf16 [2][batch * Q][heads * head_dim], hi then lo plane."""
    lib = load()
    code = lib.orthrus_attention(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_blk), _ptr(v_blk), _ptr(lens), batch,
                                 n_kv_heads, group, Q, head_dim, capacity, blk_stride, mode, _ptr(out),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
                                 _stream(stream))
    _check("orthrus_attention", code)


def attention_workspace_bytes(batch, n_kv_heads, group, Q, head_dim, capacity) -> int:
    return load().orthrus_attention_workspace_bytes(batch, n_kv_heads, group, Q, head_dim, capacity)


def linear(X, W, Y, workspace, status, stream=None):
    lib = load()
    M, Kd = X.shape
    N = W.shape[0]
    code = lib.orthrus_linear(_ptr(X), _ptr(W), _ptr(Y), M, N, Kd, _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _ptr(status), _stream(stream))
    _check("orthrus_linear", code)


def linear_noalloc(X, W, Y, status=None, stream=None):
    """orthrus_linear without a workspace: scratch in the library's static device array."""
    lib = load()
    M, Kd = X.shape
    N = W.shape[0]
    code = lib.orthrus_linear_noalloc(_ptr(X), _ptr(W), _ptr(Y), M, N, Kd, _ptr(status), _stream(stream))
    _check("orthrus_linear_noalloc", code)


def sample_tokens(logits, temperature, uniforms, out, status=None, stream=None):
    """out[r] ~ softmax(logits[r] / temperature) drawn with uniforms[r] (device fp32 [rows][vocab])."""
    rows, vocab = logits.shape
    code = load().orthrus_sample_tokens(_ptr(logits), rows, vocab, float(temperature), _ptr(uniforms), _ptr(out),
                                        _ptr(status), _stream(stream))
    _check("orthrus_sample_tokens", code)


def accept_stats(batch: int):
    """Zeroed acceptance counts of `batch` sequences (host memory)."""
    return (AcceptStats * batch)()


def accept_stats_update(stats, accept_len, K: int, decay: float = 1.0):
    """Fold one step's host accept lengths (ints) into `stats`."""
    n = len(accept_len)
    arr = (C.c_int32 * n)(*[int(a) for a in accept_len])
    _check("orthrus_accept_stats_update", load().orthrus_accept_stats_update(stats, arr, n, K, float(decay)))


def accept_rate(stats, b: int = 0) -> float:
    return float(load().orthrus_accept_rate(C.byref(stats[b])))


def choose_block_size(stats, ks, step_ms) -> int:
    """The K of `ks` that commits the most tokens per ms (measured step times `step_ms`)."""
    n = len(ks)
    k_arr = (C.c_int32 * n)(*[int(k) for k in ks])
    t_arr = (C.c_float * n)(*[float(t) for t in step_ms])
    k = load().orthrus_choose_block_size(stats, len(stats), k_arr, t_arr, n)
    if k < 0:
        raise OrthrusError("orthrus_choose_block_size", ERR_ARG)
    return int(k)


def linear_workspace_bytes(M, N, Kd) -> int:
    return load().orthrus_linear_workspace_bytes(M, N, Kd)


# ---- a plan with its device buffers --------------------------------------------------------------

_LAYER_FIELDS = [("attn_norm", "attn_norm"), ("mlp_norm", "mlp_norm"), ("w_qkv", "w_qkv"), ("w_o", "w_o"),
                 ("q_norm", "q_norm"), ("k_norm", "k_norm"), ("w_gate_up", "w_gate_up"), ("w_down", "w_down"),
                 ("wd_qkv", "wd_qkv"), ("wd_o", "wd_o"), ("wd_q_norm", "wd_q_norm"), ("wd_k_norm", "wd_k_norm")]


def upload(arr: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bits -> torch.bfloat16 on the device; float arrays -> float32."""
    if arr.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32)).to(device)


class DeviceModel:
    """Weights, KV cache, workspace and plan of one Orthrus model on the current GPU.

    ``weights`` maps the tensor names of ``synth.tensor_specs`` to host arrays
    (uint16 bf16 bits or float32 gains), or to device tensors already uploaded.
    """

    def __init__(self, shape, weights: dict, batch: int, capacity: int, max_block: int, max_rows: int | None = None,
                 device="cuda"):
        lib = load()
        self.shape = shape
        self.batch, self.capacity, self.max_block = batch, capacity, max_block
        self.max_rows = max_rows or batch * (max_block + 1)
        self.cfg = make_config(shape)
        self.dev = {k: (v if isinstance(v, torch.Tensor) else upload(v, device)) for k, v in weights.items()}
        L, Hkv, d = shape.n_layers, shape.n_kv_heads, shape.head_dim
        # K/V cache: bf16 values held in the fp16 encoding (the attention MMAs take fp16 operands)
        self.k_cache = torch.zeros((L, batch, Hkv, capacity, d), dtype=torch.float16, device=device)
        self.v_cache = torch.zeros_like(self.k_cache)
        self.lens = torch.zeros(batch, dtype=torch.int32, device=device)
        self._arrays = {}
        wfields = {}
        for field, key in _LAYER_FIELDS:
            arr = (C.c_void_p * L)(*[self.dev[f"l{l}.{key}"].data_ptr() for l in range(L)])
            self._arrays[field] = arr
            wfields[field] = C.cast(arr, _PP)
        self.weights = Weights(self.dev["embed"].data_ptr(), self.dev["final_norm"].data_ptr(),
                               self.dev["lm_head"].data_ptr(), **wfields)
        self.cache = Cache(self.k_cache.data_ptr(), self.v_cache.data_ptr(), self.lens.data_ptr(), batch, capacity)
        self.ws_bytes = lib.orthrus_workspace_bytes(C.byref(self.cfg), batch, capacity, max_block, self.max_rows)
        if self.ws_bytes == 0:
            raise OrthrusError("orthrus_workspace_bytes", ERR_ARG)
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)
        nplan = lib.orthrus_plan_bytes(C.byref(self.cfg))
        self.plan = C.create_string_buffer(nplan)
        _check("orthrus_plan_init",
               lib.orthrus_plan_init(self.plan, nplan, C.byref(self.cfg), C.byref(self.weights), C.byref(self.cache),
                                     max_block, self.max_rows, _ptr(self.workspace), self.ws_bytes, _stream()))
        self.status_addr = lib.orthrus_status_ptr(self.plan)
        off = self.status_addr - self.workspace.data_ptr()
        self.status = self.workspace[off:off + 4].view(torch.int32)
        self.block_scratch_bytes = lib.orthrus_block_scratch_bytes(C.byref(self.cfg), batch, max_block)

    # -- calls ----------------------------------------------------------------------------------
    def prefill(self, tokens: torch.Tensor, prompt_len, pending: torch.Tensor, stream=None):
        """tokens: device int32 [batch][max_prompt]; prompt_len: host ints."""
        pl = (C.c_int32 * self.batch)(*[int(x) for x in prompt_len])
        _check("orthrus_prefill", load().orthrus_prefill(self.plan, _ptr(tokens), pl, tokens.shape[1], _ptr(pending),
                                                         _stream(stream)))

    def draft_block(self, pending, K, draft, logits=None, stream=None):
        _check("orthrus_draft_block",
               load().orthrus_draft_block(self.plan, _ptr(pending), K, _ptr(draft), _ptr(logits), _stream(stream)))

    def verify_block(self, pending, draft, K, ar_argmax, logits=None, stream=None):
        _check("orthrus_verify_block",
               load().orthrus_verify_block(self.plan, _ptr(pending), _ptr(draft), K, _ptr(ar_argmax), _ptr(logits),
                                           _stream(stream)))

    def accept_commit(self, pending, draft, ar_argmax, K, accept_len, committed, poison_dead=False, stream=None):
        _check("orthrus_accept_commit",
               load().orthrus_accept_commit(self.plan, _ptr(pending), _ptr(draft), _ptr(ar_argmax), K, _ptr(accept_len),
                                            _ptr(committed), int(bool(poison_dead)), _stream(stream)))

    def decode_step(self, pending, K, planted, accept_len, committed, stream=None):
        _check("orthrus_decode_step",
               load().orthrus_decode_step(self.plan, _ptr(pending), K, _ptr(planted), _ptr(accept_len),
                                          _ptr(committed), _stream(stream)))

    def draft_refine(self, pending, prev_draft, K, draft, logits=None, stream=None):
        _check("orthrus_draft_refine",
               load().orthrus_draft_refine(self.plan, _ptr(pending), _ptr(prev_draft), K, _ptr(draft), _ptr(logits),
                                           _stream(stream)))

    def decode_step_ex(self, pending, K, draft_steps, planted, accept_len, committed, stream=None):
        _check("orthrus_decode_step_ex",
               load().orthrus_decode_step_ex(self.plan, _ptr(pending), K, draft_steps, _ptr(planted),
                                             _ptr(accept_len), _ptr(committed), _stream(stream)))

    def accept_sample(self, pending, draft, draft_logits, verify_logits, K, temperature, u_accept, u_final,
                      accept_len, committed, stream=None):
        _check("orthrus_accept_sample",
               load().orthrus_accept_sample(self.plan, _ptr(pending), _ptr(draft), _ptr(draft_logits),
                                            _ptr(verify_logits), K, float(temperature), _ptr(u_accept),
                                            _ptr(u_final), _ptr(accept_len), _ptr(committed), _stream(stream)))

    def decode_step_sampled(self, pending, K, temperature, u_draft, u_accept, u_final, draft_logits, verify_logits,
                            accept_len, committed, stream=None):
        _check("orthrus_decode_step_sampled",
               load().orthrus_decode_step_sampled(self.plan, _ptr(pending), K, float(temperature), _ptr(u_draft),
                                                  _ptr(u_accept), _ptr(u_final), _ptr(draft_logits),
                                                  _ptr(verify_logits), _ptr(accept_len), _ptr(committed),
                                                  _stream(stream)))

    def clear_status(self, stream=None):
        _check("orthrus_clear_status", load().orthrus_clear_status(self.plan, _stream(stream)))

    def launches_per_step(self, K) -> int:
        return load().orthrus_decode_step_launches(self.plan, K)

    def trace(self, events, kinds, count):
        """events: ctypes array of cudaEvent_t handles (or None to stop); kinds/count: ctypes int32 arrays."""
        if events is None:
            _check("orthrus_trace", load().orthrus_trace(self.plan, None, None, 0, None))
        else:
            _check("orthrus_trace", load().orthrus_trace(self.plan, events, kinds, len(events), count))

    def timeline(self, buf):
        """buf: device uint8/int64 tensor of timeline_bytes() bytes, or None to stop."""
        if buf is None:
            _check("orthrus_timeline", load().orthrus_timeline(self.plan, None, 0))
        else:
            _check("orthrus_timeline",
                   load().orthrus_timeline(self.plan, _ptr(buf), buf.numel() * buf.element_size()))

    def timeline_bytes(self) -> int:
        return load().orthrus_timeline_bytes(self.plan)

    def read_status(self) -> int:
        return int(self.status.item())
