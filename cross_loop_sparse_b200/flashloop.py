"""Thin Python binding of libflashloop.so (the C ABI in include/flashloop.h).

Argument marshalling only: every step of the sublayer runs in the library's
CUDA kernels.  PyTorch supplies device memory and the current stream.  If
the shared library is missing this module raises at import time; there is
no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import re
from ctypes import POINTER, c_float, c_int32, c_size_t, c_void_p

import torch

MAX_LOOPS = 16
GROUP = 32
PAPER_GROUP = 64   # the pages' cache setting: groups of 64 and a 64-token bf16 tail
PAPER_TAIL = 64
_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libflashloop.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "flashloop.h")

STATUS = {0: "FLASHLOOP_OK", -1: "FLASHLOOP_ERR_INVALID_ARG", -2: "FLASHLOOP_ERR_UNSUPPORTED",
          -3: "FLASHLOOP_ERR_CUDA", -4: "FLASHLOOP_ERR_DEVICE", -5: "FLASHLOOP_ERR_ARCH"}


class FlashLoopError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} returned {status} ({STATUS.get(status, 'unknown')})")


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m cross_loop_sparse_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)


# ----------------------------------------------------------------------------- structs
class Params(ctypes.Structure):
    _fields_ = [("seq", c_int32), ("d_model", c_int32), ("n_heads", c_int32), ("head_dim", c_int32),
                ("n_loops", c_int32), ("batch", c_int32), ("tau", c_float), ("rope_theta", c_float),
                ("topk", c_int32 * MAX_LOOPS), ("bits", c_int32 * MAX_LOOPS),
                ("capacity", c_int32 * MAX_LOOPS), ("gate_topk", c_int32), ("fixed_mass", c_int32),
                ("attn_pairs", c_int32), ("kv_scheme", c_int32)]

    @classmethod
    def from_config(cls, cfg, capacity=None, topk=None, tau=None, seq=None, token_budgets=None,
                    fixed_mass=False, kv_scheme="spec"):
        """Params of a workload.Config; capacities default to S (no overflow possible).
        token_budgets (per loop) selects top-k token retention with those budgets;
        fixed_mass selects the fixed-mass form of the sparse update; attn_pairs
        (reserved) stays 0."""
        p = cls()
        p.kv_scheme = {"spec": 0, "paper": 1}[kv_scheme]
        p.fixed_mass = 1 if fixed_mass else 0
        p.attn_pairs = 0
        p.seq = cfg.seq if seq is None else seq
        p.d_model, p.n_heads, p.head_dim = cfg.d_model, cfg.n_heads, cfg.head_dim
        p.n_loops, p.batch = cfg.n_loops, (cfg.batch if cfg.decode else 1)
        p.tau = cfg.tau if tau is None else tau
        p.rope_theta = cfg.rope_theta
        ks = cfg.k_per_loop() if topk is None else list(topk)
        for r in range(cfg.n_loops):
            p.topk[r] = ks[r]
            p.bits[r] = cfg.bits[r]
            p.capacity[r] = p.seq if capacity is None else capacity[r]
        if token_budgets is not None:
            p.gate_topk = 1
            for r in range(1, cfg.n_loops):
                p.capacity[r] = token_budgets[r]
        return p


class KV(ctypes.Structure):
    _fields_ = [("base_codes", c_void_p), ("base_scales", c_void_p),
                ("res_codes", c_void_p * MAX_LOOPS), ("res_scales", c_void_p * MAX_LOOPS)]


class PaperKV(ctypes.Structure):
    _fields_ = [("codes", c_void_p * MAX_LOOPS), ("scale", c_void_p * MAX_LOOPS),
                ("minv", c_void_p * MAX_LOOPS), ("tail", c_void_p * MAX_LOOPS)]


class StateC(ctypes.Structure):
    _fields_ = [("k", KV), ("v", KV), ("active", c_void_p * MAX_LOOPS), ("slot", c_void_p * MAX_LOOPS),
                ("n_active", c_void_p), ("q", c_void_p * 3), ("m", c_void_p * 3), ("Z", c_void_p * 3),
                ("N", c_void_p * 3), ("colmass", c_void_p * 2), ("cols", c_void_p * MAX_LOOPS),
                ("O", c_void_p), ("Y", c_void_p), ("rope_cs", c_void_p), ("err_word", c_void_p),
                ("workspace", c_void_p), ("workspace_bytes", c_size_t), ("G", c_void_p * 3),
                ("paper_k", POINTER(PaperKV)), ("paper_v", POINTER(PaperKV))]


class DecodeStateC(ctypes.Structure):
    _fields_ = [("k", KV), ("v", KV), ("rope_cs", c_void_p), ("q", c_void_p * 3), ("m", c_void_p * 3),
                ("Z", c_void_p * 3), ("N", c_void_p * 3), ("probs", c_void_p), ("cols", c_void_p),
                ("O", c_void_p), ("Y", c_void_p), ("err_word", c_void_p), ("workspace", c_void_p),
                ("workspace_bytes", c_size_t)]


# ----------------------------------------------------------------------------- prototypes
_P = POINTER(Params)
_S = POINTER(StateC)
_D = POINTER(DecodeStateC)
_V = c_void_p
_I = c_int32
_SIG = {
    "flashloop_workspace_bytes": (c_size_t, [_P]),
    "flashloop_cache_bytes": (c_size_t, [_P, _V]),
    "flashloop_rope_table": (_I, [_P, _I, _V, _V]),
    "flashloop_gate": (_I, [_P, _V, _V, _V, _V, _I, _V, _V, _V, _I, _V, _V, _V]),
    "flashloop_gate_noalloc": (_I, [_P, _V, _V, _V, _V, _I, _V, _V, _V, _I, _V, _V]),
    "flashloop_gate_topk": (_I, [_P, _V, _V, _V, _V, _I, _I, _V, _V, _V, _I, _V, _V, _V]),
    "flashloop_qkv_gathered": (_I, [_P, _V, _V, _V, _I, _V, _V, _V, _V, _V, _V]),
    "flashloop_kv_quant_residual": (_I, [_P, _I, _V, _V, _V, _V, _S, _V]),
    "flashloop_qkv_quant": (_I, [_P, _I, _V, _V, _V, _V, _S, _V, _V]),
    "flashloop_paper_kv_quant": (_I, [_P, _I, _V, _V, _V, _V, _S, _V]),
    "flashloop_topk_columns": (_I, [_P, _V, _V, _I, _I, _V, _V]),
    "flashloop_selcol_dequant": (_I, [_P, _I, _S, _V]),
    "flashloop_sparse_attn_update": (_I, [_P, _I, _S, _I, _V]),
    "flashloop_out_proj": (_I, [_P, _V, _V, _V, _I, _V, _V, _V]),
    "flashloop_loop_step": (_I, [_P, _I, _V, _V, _V, _V, _S, _V]),
    "flashloop_kv_step": (_I, [_P, _I, _V, _V, _V, _S, _V]),
    "flashloop_kv_workspace_bytes": (c_size_t, [_P]),
    "flashloop_decode_workspace_bytes": (c_size_t, [_P]),
    "flashloop_decode_attn": (_I, [_P, _I, _S, _D, _V]),
    "flashloop_decode_step": (_I, [_P, _I, _V, _V, _V, _S, _D, _V]),
    "flashloop_decode_qkv": (_I, [_P, _I, _V, _V, _D, _V]),
    "flashloop_decode_select": (_I, [_P, _D, _V]),
    "flashloop_decode_out": (_I, [_P, _V, _D, _V]),
    "flashloop_selection_loop": (_I, [_P, _I]),
    "flashloop_check_error_word": (_I, [_V, POINTER(c_int32), _V]),
    "flashloop_selftest_bounded_wait": (_I, [_I, _V, _V]),
    "flashloop_status_string": (ctypes.c_char_p, [_I]),
}
for _name, (_res, _args) in _SIG.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def header_functions():
    """Names of the functions include/flashloop.h declares."""
    text = open(HEADER_PATH).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(flashloop_[a-z_0-9]+)\s*\(",
                                 text, flags=re.M)))


def exported_symbols():
    return {n for n in header_functions() if hasattr(_lib, n)}


# ----------------------------------------------------------------------------- marshalling
def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(name, rc):
    if rc != 0:
        raise FlashLoopError(name, rc)
    return rc


def flashloop_workspace_bytes(params: Params) -> int:
    return int(_lib.flashloop_workspace_bytes(ctypes.byref(params)))


def flashloop_cache_bytes(params: Params, n_per_loop) -> int:
    arr = (c_int32 * MAX_LOOPS)(*list(n_per_loop))
    return int(_lib.flashloop_cache_bytes(ctypes.byref(params), ctypes.cast(arr, c_void_p)))


def flashloop_selection_loop(params: Params, loop: int) -> int:
    return int(_lib.flashloop_selection_loop(ctypes.byref(params), loop))


def flashloop_status_string(status: int) -> str:
    return _lib.flashloop_status_string(status).decode()


def flashloop_rope_table(params, n_pos, cs, stream=None):
    return _check("flashloop_rope_table",
                  _lib.flashloop_rope_table(ctypes.byref(params), n_pos, _ptr(cs), _stream(stream)))


def flashloop_gate(params, x_cur, x_prev, prev_active, n_prev, prev_capacity, active_out, slot_out,
                   n_active_out, out_capacity, workspace, err_word, stream=None):
    return _check("flashloop_gate", _lib.flashloop_gate(
        ctypes.byref(params), _ptr(x_cur), _ptr(x_prev), _ptr(prev_active), _ptr(n_prev),
        prev_capacity, _ptr(active_out), _ptr(slot_out), _ptr(n_active_out), out_capacity,
        _ptr(workspace), _ptr(err_word), _stream(stream)))


def flashloop_gate_topk(params, x_cur, x_prev, prev_active, n_prev, prev_capacity, budget, active_out,
                        slot_out, n_active_out, out_capacity, workspace, err_word, stream=None):
    return _check("flashloop_gate_topk", _lib.flashloop_gate_topk(
        ctypes.byref(params), _ptr(x_cur), _ptr(x_prev), _ptr(prev_active), _ptr(n_prev), prev_capacity,
        budget, _ptr(active_out), _ptr(slot_out), _ptr(n_active_out), out_capacity, _ptr(workspace),
        _ptr(err_word), _stream(stream)))


def flashloop_gate_noalloc(params, x_cur, x_prev, prev_active, n_prev, prev_capacity, active_out,
                           slot_out, n_active_out, out_capacity, err_word, stream=None):
    """flashloop_gate without a workspace: for callers that cannot allocate;
    its scratch is a fixed device array inside the library (see the header)."""
    return _check("flashloop_gate_noalloc", _lib.flashloop_gate_noalloc(
        ctypes.byref(params), _ptr(x_cur), _ptr(x_prev), _ptr(prev_active), _ptr(n_prev),
        prev_capacity, _ptr(active_out), _ptr(slot_out), _ptr(n_active_out), out_capacity,
        _ptr(err_word), _stream(stream)))


def flashloop_qkv_gathered(params, x, active, n_active, capacity, w_qkv, rope_cs, q_out, k_out,
                           v_out, stream=None):
    return _check("flashloop_qkv_gathered", _lib.flashloop_qkv_gathered(
        ctypes.byref(params), _ptr(x), _ptr(active), _ptr(n_active), capacity, _ptr(w_qkv),
        _ptr(rope_cs), _ptr(q_out), _ptr(k_out), _ptr(v_out), _stream(stream)))


def flashloop_kv_quant_residual(params, loop, k_new, v_new, active, n_active, state, stream=None):
    return _check("flashloop_kv_quant_residual", _lib.flashloop_kv_quant_residual(
        ctypes.byref(params), loop, _ptr(k_new), _ptr(v_new), _ptr(active), _ptr(n_active),
        ctypes.byref(state.c), _stream(stream)))


def flashloop_qkv_quant(params, loop, x, active, n_active, w_qkv, state, q_out, stream=None):
    return _check("flashloop_qkv_quant", _lib.flashloop_qkv_quant(
        ctypes.byref(params), loop, _ptr(x), _ptr(active), _ptr(n_active), _ptr(w_qkv),
        ctypes.byref(state.c), _ptr(q_out), _stream(stream)))


def flashloop_paper_kv_quant(params, loop, k_new, v_new, active, n_active, state, stream=None):
    return _check("flashloop_paper_kv_quant", _lib.flashloop_paper_kv_quant(
        ctypes.byref(params), loop, _ptr(k_new), _ptr(v_new), _ptr(active), _ptr(n_active),
        ctypes.byref(state.c), _stream(stream)))


def flashloop_topk_columns(params, mass, candidates, n_cand, k, out, stream=None):
    return _check("flashloop_topk_columns", _lib.flashloop_topk_columns(
        ctypes.byref(params), _ptr(mass), _ptr(candidates), n_cand, k, _ptr(out), _stream(stream)))


def flashloop_selcol_dequant(params, loop, state, stream=None):
    return _check("flashloop_selcol_dequant", _lib.flashloop_selcol_dequant(
        ctypes.byref(params), loop, ctypes.byref(state.c), _stream(stream)))


def flashloop_sparse_attn_update(params, loop, state, want_colmass=0, stream=None):
    return _check("flashloop_sparse_attn_update", _lib.flashloop_sparse_attn_update(
        ctypes.byref(params), loop, ctypes.byref(state.c), int(want_colmass), _stream(stream)))


def flashloop_out_proj(params, o, active, n_active, capacity, w_o, y, stream=None):
    return _check("flashloop_out_proj", _lib.flashloop_out_proj(
        ctypes.byref(params), _ptr(o), _ptr(active), _ptr(n_active), capacity, _ptr(w_o), _ptr(y),
        _stream(stream)))


def flashloop_loop_step(params, loop, x_cur, x_prev, w_qkv, w_o, state, stream=None):
    return _check("flashloop_loop_step", _lib.flashloop_loop_step(
        ctypes.byref(params), loop, _ptr(x_cur), _ptr(x_prev), _ptr(w_qkv), _ptr(w_o),
        ctypes.byref(state.c), _stream(stream)))


def flashloop_kv_step(params, loop, x_cur, x_prev, w_qkv, state, stream=None):
    return _check("flashloop_kv_step", _lib.flashloop_kv_step(
        ctypes.byref(params), loop, _ptr(x_cur), _ptr(x_prev), _ptr(w_qkv), ctypes.byref(state.c),
        _stream(stream)))


def flashloop_kv_workspace_bytes(params: Params) -> int:
    return int(_lib.flashloop_kv_workspace_bytes(ctypes.byref(params)))


def flashloop_decode_workspace_bytes(params: Params) -> int:
    return int(_lib.flashloop_decode_workspace_bytes(ctypes.byref(params)))


def flashloop_decode_attn(params, loop, ctx, dstate, stream=None):
    return _check("flashloop_decode_attn", _lib.flashloop_decode_attn(
        ctypes.byref(params), loop, ctypes.byref(ctx.c), ctypes.byref(dstate.c), _stream(stream)))


def flashloop_decode_qkv(params, loop, x_tok, w_qkv, dstate, stream=None):
    return _check("flashloop_decode_qkv", _lib.flashloop_decode_qkv(
        ctypes.byref(params), loop, _ptr(x_tok), _ptr(w_qkv), ctypes.byref(dstate.c), _stream(stream)))


def flashloop_decode_select(params, dstate, stream=None):
    return _check("flashloop_decode_select", _lib.flashloop_decode_select(
        ctypes.byref(params), ctypes.byref(dstate.c), _stream(stream)))


def flashloop_decode_out(params, w_o, dstate, stream=None):
    return _check("flashloop_decode_out", _lib.flashloop_decode_out(
        ctypes.byref(params), _ptr(w_o), ctypes.byref(dstate.c), _stream(stream)))


def flashloop_decode_step(params, loop, x_tok, w_qkv, w_o, ctx, dstate, stream=None):
    return _check("flashloop_decode_step", _lib.flashloop_decode_step(
        ctypes.byref(params), loop, _ptr(x_tok), _ptr(w_qkv), _ptr(w_o), ctypes.byref(ctx.c),
        ctypes.byref(dstate.c), _stream(stream)))


def flashloop_selftest_bounded_wait(kind, err_word, stream=None):
    return _check("flashloop_selftest_bounded_wait", _lib.flashloop_selftest_bounded_wait(
        int(kind), _ptr(err_word), _stream(stream)))


def flashloop_check_error_word(err_word, stream=None):
    """Returns the device error code (0 = none); synchronises the stream."""
    code = c_int32(0)
    rc = _lib.flashloop_check_error_word(_ptr(err_word), ctypes.byref(code), _stream(stream))
    if rc not in (0, -4):
        raise FlashLoopError("flashloop_check_error_word", rc)
    return int(code.value)


# ----------------------------------------------------------------------------- state
class FlashLoopState:
    """Caller-owned device buffers of one sequence (torch tensors) and the
    C struct that points at them.  Allocation is the only work done here."""

    def __init__(self, params: Params, device="cuda", kv_only=False, rope_period=None):
        """kv_only: only what flashloop_kv_step touches (caches, active lists,
        slot maps, counts, the gate's scratch, RoPE table, error word).
        rope_period: positions restart every rope_period rows (sequences laid
        end to end, as a decode context is)."""
        self.params = params
        S, H, dh, d, R = params.seq, params.n_heads, params.head_dim, params.d_model, params.n_loops
        self.device = device
        dev = torch.device(device)
        z = lambda shape, dt: torch.zeros(shape, dtype=dt, device=dev)  # noqa: E731
        self.t = {}
        c = StateC()
        self._paper = []
        if params.kv_scheme == 1:
            # the pages' cache setting: per loop INT4 codes, fp16 scales and minima, bf16 tail
            tail = min(PAPER_TAIL, S)
            body = S - tail
            for name in ("k", "v"):
                kv = PaperKV()
                for r in range(1, R + 1):
                    rows = max(body if r == 1 else params.capacity[r - 1], 1)
                    groups = (rows + PAPER_GROUP - 1) // PAPER_GROUP
                    gshape = (groups, H, dh) if name == "k" else (rows, H, dh // PAPER_GROUP)
                    self.t[f"p{name}_codes{r}"] = z((rows, H, dh // 2), torch.uint8)
                    self.t[f"p{name}_scale{r}"] = z(gshape, torch.float16)
                    self.t[f"p{name}_min{r}"] = z(gshape, torch.float16)
                    self.t[f"p{name}_tail{r}"] = z((max(tail, 1), H, dh), torch.bfloat16)
                    kv.codes[r - 1] = self.t[f"p{name}_codes{r}"].data_ptr()
                    kv.scale[r - 1] = self.t[f"p{name}_scale{r}"].data_ptr()
                    kv.minv[r - 1] = self.t[f"p{name}_min{r}"].data_ptr()
                    kv.tail[r - 1] = self.t[f"p{name}_tail{r}"].data_ptr()
                self._paper.append(kv)
            c.paper_k = ctypes.pointer(self._paper[0])
            c.paper_v = ctypes.pointer(self._paper[1])
        for name, kv in (("k", c.k), ("v", c.v)) if params.kv_scheme == 0 else ():
            base = z((S, H, dh), torch.int8)
            bs = z((S, H, dh // GROUP), torch.float16)
            self.t[f"{name}_base"], self.t[f"{name}_base_s"] = base, bs
            kv.base_codes, kv.base_scales = base.data_ptr(), bs.data_ptr()
            for r in range(2, R + 1):
                cap, b = params.capacity[r - 1], params.bits[r - 1]
                codes = z((cap, H, dh * b // 8), torch.uint8)
                sc = z((cap, H, dh // GROUP), torch.float16)
                self.t[f"{name}_res{r}"], self.t[f"{name}_res{r}_s"] = codes, sc
                kv.res_codes[r - 1], kv.res_scales[r - 1] = codes.data_ptr(), sc.data_ptr()
        for r in range(2, R + 1):
            act = z((params.capacity[r - 1],), torch.int32)
            slot = torch.full((S,), -1, dtype=torch.int32, device=dev)
            self.t[f"active{r}"], self.t[f"slot{r}"] = act, slot
            c.active[r - 1], c.slot[r - 1] = act.data_ptr(), slot.data_ptr()
        self.t["n_active"] = z((MAX_LOOPS,), torch.int32)
        c.n_active = self.t["n_active"].data_ptr()
        self.t["rope_cs"] = z((S, dh // 2, 2), torch.float32)
        self.t["err"] = z((1,), torch.int32)
        c.rope_cs, c.err_word = self.t["rope_cs"].data_ptr(), self.t["err"].data_ptr()
        self.c = c
        if rope_period is None:
            flashloop_rope_table(params, S, self.t["rope_cs"])
        else:
            assert S % rope_period == 0
            one = z((rope_period, dh // 2, 2), torch.float32)
            flashloop_rope_table(params, rope_period, one)
            self.t["rope_cs"].copy_(one.repeat(S // rope_period, 1, 1))
        if kv_only:
            ws = flashloop_kv_workspace_bytes(params)
            self.t["workspace"] = z((max(ws, 256),), torch.uint8)
            c.workspace, c.workspace_bytes = self.t["workspace"].data_ptr(), ws
            return
        for i in range(3):
            self.t[f"q{i}"] = z((S, d), torch.bfloat16)
            self.t[f"m{i}"] = z((H, S), torch.float32)
            self.t[f"Z{i}"] = z((H, S), torch.float32)
            self.t[f"N{i}"] = z((H, S, dh), torch.float32)
            c.q[i], c.m[i] = self.t[f"q{i}"].data_ptr(), self.t[f"m{i}"].data_ptr()
            c.Z[i], c.N[i] = self.t[f"Z{i}"].data_ptr(), self.t[f"N{i}"].data_ptr()
            if params.fixed_mass:
                self.t[f"G{i}"] = z((H, S), torch.float32)
                c.G[i] = self.t[f"G{i}"].data_ptr()
        for i in range(2):
            self.t[f"colmass{i}"] = z((H, S), torch.float32)
            c.colmass[i] = self.t[f"colmass{i}"].data_ptr()
        for r in range(2, R + 1):
            if flashloop_selection_loop(params, r) == r:
                self.t[f"cols{r}"] = z((H, params.topk[r - 1]), torch.int32)
                c.cols[r - 1] = self.t[f"cols{r}"].data_ptr()
        self.t["O"] = z((S, d), torch.bfloat16)
        self.t["Y"] = z((S, d), torch.bfloat16)
        ws = flashloop_workspace_bytes(params)
        self.t["workspace"] = z((max(ws, 256),), torch.uint8)
        c.O, c.Y = self.t["O"].data_ptr(), self.t["Y"].data_ptr()
        c.workspace, c.workspace_bytes = self.t["workspace"].data_ptr(), ws

    def __getitem__(self, key):
        return self.t[key]

    def cols_for_loop(self, r):
        return self.t[f"cols{flashloop_selection_loop(self.params, r)}"]

    def q_slot(self, r):
        return 0 if r == 1 else 1 + (r % 2)

    def error_code(self, stream=None):
        return flashloop_check_error_word(self.t["err"], stream)


# ----------------------------------------------------------------------------- decode
def decode_context_params(params: Params, capacity=None) -> Params:
    """Params of the B contexts of a decode laid end to end (seq = B*S), the
    layout flashloop_decode_attn reads; capacities default to B*S."""
    p = Params()
    ctypes.pointer(p)[0] = params
    p.seq = params.batch * params.seq
    p.batch = 1
    for r in range(params.n_loops):
        p.capacity[r] = p.seq if capacity is None else capacity[r]
    return p


class DecodeContext(FlashLoopState):
    """Caches of the B contexts of a decode (kv-only state of B*S rows, RoPE
    positions restarting at every sequence)."""

    def __init__(self, params: Params, device="cuda", capacity=None):
        self.dec_params = params
        super().__init__(decode_context_params(params, capacity), device, kv_only=True,
                         rope_period=params.seq)

    def prepare(self, xs, w_qkv, stream=None):
        """KV path of loops 1..R: xs[r-1] is bf16 [B*S, d] (the contexts of loop r)."""
        p = self.params
        for r in range(1, p.n_loops + 1):
            flashloop_kv_step(p, r, xs[r - 1], xs[r - 2] if r > 1 else None, w_qkv, self, stream)


class DecodeState:
    """Caller-owned device buffers of a decode step (B sequences, one token
    each at position S) and the C struct that points at them."""

    def __init__(self, params: Params, device="cuda"):
        self.params = params
        S, H, dh, d, R, B = (params.seq, params.n_heads, params.head_dim, params.d_model, params.n_loops,
                             params.batch)
        dev = torch.device(device)
        z = lambda shape, dt: torch.zeros(shape, dtype=dt, device=dev)  # noqa: E731
        self.t = {}
        c = DecodeStateC()
        for name, kv in (("k", c.k), ("v", c.v)):
            base = z((B, H, dh), torch.int8)
            bs = z((B, H, dh // GROUP), torch.float16)
            self.t[f"{name}_base"], self.t[f"{name}_base_s"] = base, bs
            kv.base_codes, kv.base_scales = base.data_ptr(), bs.data_ptr()
            for r in range(2, R + 1):
                b = params.bits[r - 1]
                codes = z((B, H, dh * b // 8), torch.uint8)
                sc = z((B, H, dh // GROUP), torch.float16)
                self.t[f"{name}_res{r}"], self.t[f"{name}_res{r}_s"] = codes, sc
                kv.res_codes[r - 1], kv.res_scales[r - 1] = codes.data_ptr(), sc.data_ptr()
        for i in range(3):
            self.t[f"q{i}"] = z((B, d), torch.bfloat16)
            self.t[f"m{i}"] = z((B, H), torch.float32)
            self.t[f"Z{i}"] = z((B, H), torch.float32)
            self.t[f"N{i}"] = z((B, H, dh), torch.float32)
            c.q[i], c.m[i] = self.t[f"q{i}"].data_ptr(), self.t[f"m{i}"].data_ptr()
            c.Z[i], c.N[i] = self.t[f"Z{i}"].data_ptr(), self.t[f"N{i}"].data_ptr()
        self.t["probs"] = z((B, H, S + 1), torch.float32)
        k = params.topk[1] if R >= 2 else 1
        self.t["cols"] = z((B, H, k), torch.int32)
        self.t["O"] = z((B, d), torch.bfloat16)
        self.t["Y"] = z((B, d), torch.bfloat16)
        self.t["err"] = z((1,), torch.int32)
        table = z((S + 1, dh // 2, 2), torch.float32)
        flashloop_rope_table(params, S + 1, table)
        self.t["rope_cs"] = table[S].clone()
        ws = flashloop_decode_workspace_bytes(params)
        if ws == 0:
            raise FlashLoopError("flashloop_decode_workspace_bytes", -2)
        self.t["workspace"] = z((ws,), torch.uint8)
        c.rope_cs, c.probs, c.cols = (self.t["rope_cs"].data_ptr(), self.t["probs"].data_ptr(),
                                      self.t["cols"].data_ptr())
        c.O, c.Y, c.err_word = self.t["O"].data_ptr(), self.t["Y"].data_ptr(), self.t["err"].data_ptr()
        c.workspace, c.workspace_bytes = self.t["workspace"].data_ptr(), ws
        self.c = c

    def __getitem__(self, key):
        return self.t[key]

    def q_slot(self, r):
        return 0 if r == 1 else 1 + (r % 2)

    def error_code(self, stream=None):
        return flashloop_check_error_word(self.t["err"], stream)
