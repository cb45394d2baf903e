"""Python binding of libgptblock.so (the C ABI declared in include/gptblock.h).

Argument marshalling only: every step of the block runs in the library's CUDA
kernels.  PyTorch supplies device memory and the stream.  There is no CPU or
PyTorch fallback: if the library is missing the import of the binding raises.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgptblock.so")
MAX_LAYERS = 64

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE, ERR_BAD_INPUT = 0, -1, -2, -3, -4, -5, -6
F32, BF16, FP8_E4M3 = 0, 1, 2
FP8_GRAD_E5M2, FP8_LM_HEAD = 1, 2
WS_BLOCK_SAVED, WS_BLOCK_SCRATCH, WS_LM_HEAD, WS_STACK = 0, 1, 2, 3
DTYPES = {"f32": F32, "bf16": BF16, "fp8": FP8_E4M3}

EXPORTS = [
    "gptb_workspace_bytes", "gpt_block_forward", "gpt_block_backward", "lm_head_xent",
    "gpt_stack_step", "gptb_gemm_bf16", "gptb_device_error", "gptb_set_wait_limit_ns",
    "gptb_reset_counters", "gptb_launch_count", "gptb_set_gemm_timing", "gptb_gemm_timing",
    "gptb_error_string", "lm_head_xent_noalloc", "gptb_probe_bounded_wait",
    "gptb_adamw_step", "gptb_polar_express_workspace_bytes", "gptb_polar_express", "gptb_decode_attention",
    "gptb_muon_workspace_bytes", "gptb_muon_step", "gptb_muon_batched_workspace_bytes", "gptb_muon_step_batched",
    "gptb_gemm_bf16_batched", "gpt_stack_step_hooked", "gptb_cast_f32_bf16",
    "gptb_cast_bf16_f32", "gptb_decode_workspace_bytes", "gptb_gemm_fp8_workspace_bytes", "gptb_gemm_fp8",
]

GRADS_READY_FN = ctypes.CFUNCTYPE(None, ctypes.c_int, ctypes.c_void_p)

_vp = ctypes.c_void_p
_fp = ctypes.POINTER(ctypes.c_float)


class Config(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("T", ctypes.c_int), ("d", ctypes.c_int),
        ("n_head", ctypes.c_int), ("n_kv_head", ctypes.c_int), ("head_dim", ctypes.c_int),
        ("mlp_hidden", ctypes.c_int), ("vocab", ctypes.c_int), ("n_layer", ctypes.c_int),
        ("window", ctypes.c_int * MAX_LAYERS), ("has_ve", ctypes.c_int * MAX_LAYERS),
        ("ve_gate_ch", ctypes.c_int), ("smear_ch", ctypes.c_int), ("backout_layer", ctypes.c_int),
        ("rope_base", ctypes.c_float), ("norm_eps", ctypes.c_float), ("dtype", ctypes.c_int),
        ("fp8_flags", ctypes.c_int),
    ]


class BlockWeights(ctypes.Structure):
    _fields_ = [("w_qkv", _vp), ("w_o", _vp), ("w_fc", _vp), ("w_proj", _vp),
                ("w_ve_gate", _vp), ("ve_table", _vp), ("lambdas", _vp)]


class BlockGrads(ctypes.Structure):
    _fields_ = [("w_qkv", _vp), ("w_o", _vp), ("w_fc", _vp), ("w_proj", _vp),
                ("w_ve_gate", _vp), ("ve_table", _vp), ("lambdas", _vp)]


class ModelWeights(ctypes.Structure):
    _fields_ = [("wte", _vp), ("w_lm", _vp), ("w_smear_gate", _vp), ("smear_lambda", _vp),
                ("backout_lambda", _vp), ("layers", BlockWeights * MAX_LAYERS)]


class ModelGrads(ctypes.Structure):
    _fields_ = [("wte", _vp), ("w_lm", _vp), ("w_smear_gate", _vp), ("smear_lambda", _vp),
                ("backout_lambda", _vp), ("layers", BlockGrads * MAX_LAYERS)]


_LIB = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (raises if it was not built)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m gpt_transformer_block_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER
    lib.gptb_workspace_bytes.argtypes = [P(Config), ctypes.c_int]
    lib.gptb_workspace_bytes.restype = ctypes.c_size_t
    lib.gpt_block_forward.argtypes = [P(Config), ctypes.c_int, P(BlockWeights), _vp, _vp, _vp, _vp, _vp, _vp, _vp]
    lib.gpt_block_backward.argtypes = [P(Config), ctypes.c_int, P(BlockWeights), _vp, _vp, _vp, _vp, _vp, _vp,
                                       _vp, _vp, P(BlockGrads), _vp, _vp]
    lib.lm_head_xent.argtypes = [P(Config), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
    lib.lm_head_xent_noalloc.argtypes = [P(Config), _vp, _vp, _vp, _vp, _vp, _vp, _vp]
    lib.gpt_stack_step.argtypes = [P(Config), P(ModelWeights), _vp, _vp, _vp, P(ModelGrads), _vp, _vp]
    lib.gptb_gemm_bf16.argtypes = [_vp, ctypes.c_int, ctypes.c_longlong, _vp, ctypes.c_int, ctypes.c_longlong,
                                   _vp, ctypes.c_int, ctypes.c_longlong, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_int, _vp]
    lib.gptb_device_error.argtypes = [_vp]
    lib.gptb_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    lib.gptb_probe_bounded_wait.argtypes = [ctypes.c_ulonglong, _vp]
    lib.gptb_reset_counters.restype = None
    lib.gptb_launch_count.restype = ctypes.c_longlong
    lib.gptb_set_gemm_timing.argtypes = [ctypes.c_int]
    lib.gptb_gemm_timing.argtypes = [P(ctypes.c_double), P(ctypes.c_double), P(ctypes.c_double), P(ctypes.c_double),
                                     P(ctypes.c_longlong)]
    lib.gptb_error_string.argtypes = [ctypes.c_int]
    lib.gptb_error_string.restype = ctypes.c_char_p
    lib.gptb_adamw_step.argtypes = [_vp, _vp, _vp, _vp, _vp, ctypes.c_longlong, ctypes.c_float, ctypes.c_float,
                                    ctypes.c_float, ctypes.c_float, ctypes.c_float, ctypes.c_int, _vp]
    lib.gptb_polar_express_workspace_bytes.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.gptb_polar_express_workspace_bytes.restype = ctypes.c_size_t
    lib.gptb_polar_express.argtypes = [_vp, _vp, ctypes.c_int, ctypes.c_int, _fp, ctypes.c_int, _vp,
                                       ctypes.c_size_t, _vp]
    lib.gptb_decode_attention.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, _vp, ctypes.c_size_t, _vp]
    lib.gptb_gemm_fp8_workspace_bytes.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.gptb_gemm_fp8_workspace_bytes.restype = ctypes.c_size_t
    lib.gptb_gemm_fp8.argtypes = [_vp, ctypes.c_int, ctypes.c_longlong, _vp, ctypes.c_int, ctypes.c_longlong, _vp,
                                  ctypes.c_longlong, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp,
                                  ctypes.c_size_t, _vp]
    lib.gptb_decode_workspace_bytes.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.gptb_decode_workspace_bytes.restype = ctypes.c_size_t
    lib.gpt_stack_step_hooked.argtypes = [P(Config), P(ModelWeights), _vp, _vp, _vp, P(ModelGrads), _vp, _vp,
                                          GRADS_READY_FN, _vp]
    lib.gptb_cast_f32_bf16.argtypes = [_vp, _vp, ctypes.c_longlong, ctypes.c_float, _vp]
    lib.gptb_cast_bf16_f32.argtypes = [_vp, _vp, ctypes.c_longlong, ctypes.c_float, _vp]
    lib.gptb_muon_workspace_bytes.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.gptb_muon_workspace_bytes.restype = ctypes.c_size_t
    lib.gptb_muon_step.argtypes = [_vp, _vp, _vp, _vp, _vp, ctypes.c_int, ctypes.c_int, _fp, ctypes.c_int,
                                   ctypes.c_float, ctypes.c_float, ctypes.c_float, ctypes.c_float, _vp,
                                   ctypes.c_size_t, _vp]
    lib.gptb_muon_batched_workspace_bytes.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.gptb_muon_batched_workspace_bytes.restype = ctypes.c_size_t
    lib.gptb_muon_step_batched.argtypes = [ctypes.c_int, P(_vp), P(_vp), P(_vp), P(_vp), P(_vp), ctypes.c_int,
                                           ctypes.c_int, _fp, ctypes.c_int, ctypes.c_float, ctypes.c_float,
                                           ctypes.c_float, ctypes.c_float, _vp, ctypes.c_size_t, _vp]
    lib.gptb_gemm_bf16_batched.argtypes = [_vp, ctypes.c_int, ctypes.c_longlong, ctypes.c_longlong, _vp, ctypes.c_int,
                                           ctypes.c_longlong, ctypes.c_longlong, _vp, ctypes.c_int,
                                           ctypes.c_longlong, ctypes.c_longlong, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, _vp]
    for name in EXPORTS:
        if name not in ("gptb_workspace_bytes", "gptb_error_string", "gptb_reset_counters",
                        "gptb_launch_count", "gptb_polar_express_workspace_bytes", "gptb_muon_workspace_bytes",
                        "gptb_decode_workspace_bytes", "gptb_gemm_fp8_workspace_bytes",
                        "gptb_muon_batched_workspace_bytes"):
            getattr(lib, name).restype = ctypes.c_int
    _LIB = lib
    return lib


class GPTBError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        msg = load().gptb_error_string(code).decode()
        super().__init__(f"{what}: {msg} ({code})")


def _check(rc: int, what: str):
    if rc != OK:
        raise GPTBError(rc, what)


def ptr(t) -> int | None:
    """Device address of a tensor (None for None)."""
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def make_config(c: dict) -> Config:
    """Build the C config from a plain dict (keys of the workload presets)."""
    cfg = Config()
    for k in ("B", "T", "d", "n_head", "n_kv_head", "head_dim", "mlp_hidden", "vocab", "n_layer",
              "ve_gate_ch", "smear_ch", "backout_layer"):
        setattr(cfg, k, int(c[k]))
    L = int(c["n_layer"])
    if L > MAX_LAYERS:
        raise ValueError("too many layers")
    for i in range(L):
        cfg.window[i] = int(c["window"][i])
        cfg.has_ve[i] = int(c["has_ve"][i])
    cfg.rope_base = float(c["rope_base"])
    cfg.norm_eps = float(c["norm_eps"])
    cfg.dtype = DTYPES[c["dtype"]] if isinstance(c["dtype"], str) else int(c["dtype"])
    cfg.fp8_flags = (FP8_GRAD_E5M2 if c.get("fp8_grad") == "e5m2" else 0) | (FP8_LM_HEAD if c.get("fp8_lm_head") else 0)
    return cfg


def block_weights(lw: dict) -> BlockWeights:
    """lw: device tensors w_qkv, w_o, w_fc, w_proj, lambdas [2] fp32, optional w_ve_gate, ve_table."""
    return BlockWeights(ptr(lw["w_qkv"]), ptr(lw["w_o"]), ptr(lw["w_fc"]), ptr(lw["w_proj"]),
                        ptr(lw.get("w_ve_gate")), ptr(lw.get("ve_table")), ptr(lw["lambdas"]))


def block_grads(lg: dict) -> BlockGrads:
    return BlockGrads(ptr(lg["w_qkv"]), ptr(lg["w_o"]), ptr(lg["w_fc"]), ptr(lg["w_proj"]),
                      ptr(lg.get("w_ve_gate")), ptr(lg.get("ve_table")), ptr(lg["lambdas"]))


def model_weights(w: dict) -> ModelWeights:
    mw = ModelWeights()
    mw.wte, mw.w_lm = ptr(w["wte"]), ptr(w["w_lm"])
    mw.w_smear_gate = ptr(w.get("w_smear_gate"))
    mw.smear_lambda = ptr(w.get("smear_lambda"))
    mw.backout_lambda = ptr(w.get("backout_lambda"))
    for i, lw in enumerate(w["layers"]):
        mw.layers[i] = block_weights(lw)
    return mw


def model_grads(g: dict) -> ModelGrads:
    mg = ModelGrads()
    mg.wte, mg.w_lm = ptr(g["wte"]), ptr(g["w_lm"])
    mg.w_smear_gate = ptr(g.get("w_smear_gate"))
    mg.smear_lambda = ptr(g.get("smear_lambda"))
    mg.backout_lambda = ptr(g.get("backout_lambda"))
    for i, lg in enumerate(g["layers"]):
        mg.layers[i] = block_grads(lg)
    return mg


# ---------------------------------------------------------------- entry points

def gptb_workspace_bytes(cfg: Config, kind: int) -> int:
    return int(load().gptb_workspace_bytes(ctypes.byref(cfg), kind))


def gpt_block_forward(cfg, layer, w: BlockWeights, x, x0, idx, x_out, saved, scratch, stream=None):
    _check(load().gpt_block_forward(ctypes.byref(cfg), layer, ctypes.byref(w), ptr(x), ptr(x0), ptr(idx),
                                    ptr(x_out), ptr(saved), ptr(scratch), _stream(stream)), "gpt_block_forward")


def gpt_block_backward(cfg, layer, w: BlockWeights, x, x0, idx, saved, dx_out, dx_extra, dx, dx0_accum,
                       g: BlockGrads, scratch, stream=None):
    _check(load().gpt_block_backward(ctypes.byref(cfg), layer, ctypes.byref(w), ptr(x), ptr(x0), ptr(idx),
                                     ptr(saved), ptr(dx_out), ptr(dx_extra), ptr(dx), ptr(dx0_accum),
                                     ctypes.byref(g), ptr(scratch), _stream(stream)), "gpt_block_backward")


def lm_head_xent(cfg, h, w_lm, targets, loss_out, dh, dw_lm, ws, stream=None):
    _check(load().lm_head_xent(ctypes.byref(cfg), ptr(h), ptr(w_lm), ptr(targets), ptr(loss_out), ptr(dh),
                               ptr(dw_lm), ptr(ws), _stream(stream)), "lm_head_xent")


def lm_head_xent_noalloc(cfg, h, w_lm, targets, loss_out, dh, dw_lm, stream=None):
    """lm_head_xent with the library's own static scratch (no workspace argument)."""
    _check(load().lm_head_xent_noalloc(ctypes.byref(cfg), ptr(h), ptr(w_lm), ptr(targets), ptr(loss_out), ptr(dh),
                                       ptr(dw_lm), _stream(stream)), "lm_head_xent_noalloc")


def gpt_stack_step(cfg, w: ModelWeights, idx, targets, loss_out, g: ModelGrads, ws, stream=None):
    _check(load().gpt_stack_step(ctypes.byref(cfg), ctypes.byref(w), ptr(idx), ptr(targets), ptr(loss_out),
                                 ctypes.byref(g), ptr(ws), _stream(stream)), "gpt_stack_step")


def gpt_stack_step_hooked(cfg, w: ModelWeights, idx, targets, loss_out, g: ModelGrads, ws, ready, stream=None):
    """gpt_stack_step with ready(layer) called on this thread as each layer's
    gradients are enqueued (L-1 .. 0, then -1 for the embedding / lm_head ones)."""
    err = []

    def _cb(layer, _user):
        try:
            ready(int(layer))
        except BaseException as e:  # exceptions cannot cross the C frame: re-raised below
            err.append(e)
    cb = GRADS_READY_FN(_cb)
    rc = load().gpt_stack_step_hooked(ctypes.byref(cfg), ctypes.byref(w), ptr(idx), ptr(targets), ptr(loss_out),
                                      ctypes.byref(g), ptr(ws), _stream(stream), cb, None)
    if err:
        raise err[0]
    _check(rc, "gpt_stack_step_hooked")


def gptb_cast_f32_bf16(x, y, n, scale=1.0, stream=None):
    _check(load().gptb_cast_f32_bf16(ptr(x), ptr(y), int(n), float(scale), _stream(stream)), "gptb_cast_f32_bf16")


def gptb_cast_bf16_f32(x, y, n, scale=1.0, stream=None):
    _check(load().gptb_cast_bf16_f32(ptr(x), ptr(y), int(n), float(scale), _stream(stream)), "gptb_cast_bf16_f32")


def gptb_gemm_fp8(A, a_mn, lda, B, b_mn, ldb, C, ldc, M, N, K, a_e5m2=False, stream=None):
    """C += dequant(q(A) q(B)^T) with per-tensor FP8 casts of the bf16 operands (test entry point)."""
    import torch
    ws = torch.empty(int(load().gptb_gemm_fp8_workspace_bytes(int(M), int(N), int(K))), dtype=torch.uint8,
                     device=C.device)
    _check(load().gptb_gemm_fp8(ptr(A), int(a_mn), int(lda), ptr(B), int(b_mn), int(ldb), ptr(C), int(ldc), int(M),
                                int(N), int(K), 1 if a_e5m2 else 0, ptr(ws), ws.numel(), _stream(stream)),
           "gptb_gemm_fp8")


def gptb_gemm_bf16(A, a_mn, lda, B, b_mn, ldb, C, c_f32, ldc, M, N, K, stream=None):
    _check(load().gptb_gemm_bf16(ptr(A), int(a_mn), lda, ptr(B), int(b_mn), ldb, ptr(C), int(c_f32), ldc,
                                 M, N, K, _stream(stream)), "gptb_gemm_bf16")


def gptb_gemm_bf16_batched(A, a_mn, lda, sa, B, b_mn, ldb, sb, C, c_f32, ldc, sc, M, N, K, batch, stream=None):
    _check(load().gptb_gemm_bf16_batched(ptr(A), int(a_mn), lda, sa, ptr(B), int(b_mn), ldb, sb, ptr(C), int(c_f32),
                                         ldc, sc, M, N, K, int(batch), _stream(stream)), "gptb_gemm_bf16_batched")


def gptb_adamw_step(p, g, m, v, p_bf16, n, lr, beta1, beta2, eps, weight_decay, step, stream=None):
    """One AdamW step over n fp32 parameters in place (p, m, v); p_bf16 (or None)
    receives the bf16 copy of the new parameters."""
    _check(load().gptb_adamw_step(ptr(p), ptr(g), ptr(m), ptr(v), ptr(p_bf16) if p_bf16 is not None else None,
                                  int(n), float(lr), float(beta1), float(beta2), float(eps), float(weight_decay),
                                  int(step), _stream(stream)), "gptb_adamw_step")


def gptb_polar_express_workspace_bytes(m: int, n: int, steps: int) -> int:
    return int(load().gptb_polar_express_workspace_bytes(int(m), int(n), int(steps)))


def gptb_polar_express(G, out, m, n, coeffs, workspace, stream=None):
    """Polar Express orthogonalisation of the bf16 [m, n] matrix G into out;
    coeffs: a host sequence of (a, b, c) tuples, one per step."""
    flat = [float(x) for abc in coeffs for x in abc]
    arr = (ctypes.c_float * len(flat))(*flat)
    nbytes = workspace.numel() * workspace.element_size() if hasattr(workspace, "numel") else 0
    _check(load().gptb_polar_express(ptr(G), ptr(out), int(m), int(n), arr, len(coeffs), ptr(workspace),
                                     nbytes, _stream(stream)), "gptb_polar_express")


def gptb_muon_workspace_bytes(m: int, n: int, steps: int) -> int:
    return int(load().gptb_muon_workspace_bytes(int(m), int(n), int(steps)))


def gptb_muon_step(w, w_bf16, g, buf, v, m, n, coeffs, lr, mu, beta2, weight_decay, workspace, stream=None):
    """One Muon step (momentum, Polar Express, NorMuon, decoupled decay) on the fp32 [m, n] weight w."""
    flat = [float(x) for abc in coeffs for x in abc]
    arr = (ctypes.c_float * len(flat))(*flat)
    nbytes = workspace.numel() * workspace.element_size() if hasattr(workspace, "numel") else 0
    _check(load().gptb_muon_step(ptr(w), ptr(w_bf16), ptr(g), ptr(buf), ptr(v), int(m), int(n), arr, len(coeffs),
                                 float(lr), float(mu), float(beta2), float(weight_decay), ptr(workspace), nbytes,
                                 _stream(stream)), "gptb_muon_step")


def gptb_muon_batched_workspace_bytes(count: int, m: int, n: int, steps: int) -> int:
    return int(load().gptb_muon_batched_workspace_bytes(int(count), int(m), int(n), int(steps)))


def gptb_muon_step_batched(ws, wbs, gs, bufs, vs, m, n, coeffs, lr, mu, beta2, weight_decay, workspace, stream=None):
    """gptb_muon_step on len(ws) same-shape matrices at once (lists of tensors; wbs entries may be None)."""
    count = len(ws)
    if not (len(wbs) == len(gs) == len(bufs) == len(vs) == count):
        raise ValueError("gptb_muon_step_batched: the per-matrix lists differ in length")
    arr_t = _vp * count

    def arr(ts):
        return arr_t(*[ptr(t) if t is not None else None for t in ts])

    flat = [float(x) for abc in coeffs for x in abc]
    cf = (ctypes.c_float * len(flat))(*flat)
    nbytes = workspace.numel() * workspace.element_size() if hasattr(workspace, "numel") else 0
    _check(load().gptb_muon_step_batched(count, arr(ws), arr(wbs), arr(gs), arr(bufs), arr(vs), int(m), int(n), cf,
                                         len(coeffs), float(lr), float(mu), float(beta2), float(weight_decay),
                                         ptr(workspace), nbytes, _stream(stream)), "gptb_muon_step_batched")


def gptb_decode_workspace_bytes(B: int, H: int, T_max: int) -> int:
    return int(load().gptb_decode_workspace_bytes(int(B), int(H), int(T_max)))


def gptb_decode_attention(q, k_cache, v_cache, lens, o, lse, B, H, Hkv, T_max, window, workspace, stream=None):
    """One decode step: attention of each sequence's newest token over its KV cache."""
    nbytes = workspace.numel() * workspace.element_size() if hasattr(workspace, "numel") else 0
    _check(load().gptb_decode_attention(ptr(q), ptr(k_cache), ptr(v_cache), ptr(lens), ptr(o), ptr(lse), int(B),
                                        int(H), int(Hkv), int(T_max), int(window), ptr(workspace), nbytes,
                                        _stream(stream)), "gptb_decode_attention")


def gptb_device_error(stream=None) -> int:
    return int(load().gptb_device_error(_stream(stream)))


def gptb_probe_bounded_wait(limit_ns: int, stream=None) -> int:
    """Run the bounded-wait self-test; GPTB_ERR_TIMEOUT is the expected result."""
    return int(load().gptb_probe_bounded_wait(int(limit_ns), _stream(stream)))


def gptb_set_wait_limit_ns(ns: int):
    _check(load().gptb_set_wait_limit_ns(int(ns)), "gptb_set_wait_limit_ns")


def gptb_reset_counters():
    load().gptb_reset_counters()


def gptb_launch_count() -> int:
    return int(load().gptb_launch_count())


def gptb_set_gemm_timing(enable: bool):
    _check(load().gptb_set_gemm_timing(1 if enable else 0), "gptb_set_gemm_timing")


def gptb_gemm_timing():
    """(ms, flops, ms of e4m3 GEMMs, flops of e4m3 GEMMs, launches) since the last reset."""
    ms, fl, ms8, fl8, n = (ctypes.c_double(), ctypes.c_double(), ctypes.c_double(), ctypes.c_double(),
                           ctypes.c_longlong())
    _check(load().gptb_gemm_timing(ctypes.byref(ms), ctypes.byref(fl), ctypes.byref(ms8), ctypes.byref(fl8),
                                   ctypes.byref(n)), "gptb_gemm_timing")
    return ms.value, fl.value, ms8.value, fl8.value, n.value


from .model import GPTStack, BlockRunner, to_device_weights  # noqa: E402,F401
