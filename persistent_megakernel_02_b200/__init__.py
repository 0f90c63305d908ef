"""Persistent decode megakernel for B200 (sm_100a): Python binding.

A thin ctypes layer over the C ABI in ``include/mk.h``.  It only marshals
arguments -- every step of the decode path runs in the CUDA library
``libmk.so`` built from ``csrc/`` (``python -m persistent_megakernel_02_b200.build``).
There is no fallback: if the library is missing or a call fails, an
:class:`MkError` is raised.

PyTorch is used by callers for device memory and streams; this module only
reads ``tensor.data_ptr()`` and stream handles.
"""

from __future__ import annotations

import ctypes
import os

from .build import LIB

__all__ = ["Megakernel", "MkError", "plan_check", "version", "lib", "STATUS",
           "greedy_head_noalloc", "rope_inv_freq"]

STATUS = {
    0: "MK_OK",
    1: "MK_ERR_INVALID_ARG",
    2: "MK_ERR_UNSUPPORTED",
    3: "MK_ERR_OOM",
    4: "MK_ERR_CUDA",
    5: "MK_ERR_TIMEOUT",
    6: "MK_ERR_DEVICE_FAULT",
    7: "MK_ERR_ABORTED",
}


class MkError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)}")
        self.status = status
        self.name = STATUS.get(status, str(status))


class MkConfig(ctypes.Structure):
    _fields_ = [
        ("n_layers", ctypes.c_int32), ("hidden", ctypes.c_int32), ("n_heads", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("ffn", ctypes.c_int32),
        ("vocab", ctypes.c_int32), ("tied", ctypes.c_int32), ("rms_eps", ctypes.c_float),
        ("rope_theta", ctypes.c_float), ("rope_scaling", ctypes.c_int32),
        ("rope_factor", ctypes.c_float), ("rope_low_freq", ctypes.c_float),
        ("rope_high_freq", ctypes.c_float), ("rope_orig_max", ctypes.c_int32),
        ("max_batch", ctypes.c_int32), ("max_seq", ctypes.c_int32),
        ("kv_dtype", ctypes.c_int32),
    ]


_PP = ctypes.POINTER(ctypes.c_void_p)


class MkWeights(ctypes.Structure):
    _fields_ = [
        ("embed", ctypes.c_void_p), ("lm_head", ctypes.c_void_p), ("final_norm", ctypes.c_void_p),
        ("attn_norm", _PP), ("wq", _PP), ("wk", _PP), ("wv", _PP), ("wo", _PP),
        ("mlp_norm", _PP), ("w_gate", _PP), ("w_up", _PP), ("w_down", _PP),
    ]


class MkOptions(ctypes.Structure):
    _fields_ = [
        ("device", ctypes.c_int32), ("wait_limit_ms", ctypes.c_int32), ("n_sm", ctypes.c_int32),
        ("ring_pages", ctypes.c_int32), ("debug_fault", ctypes.c_int32),
        ("profile", ctypes.c_int32), ("dyn_percent", ctypes.c_int32),
        ("prefill_tokenwise", ctypes.c_int32), ("region_cut", ctypes.c_int32),
        ("tensor_core_units", ctypes.c_int32),
    ]


class MkPlanReport(ctypes.Structure):
    _fields_ = [
        ("n_instr_total", ctypes.c_int32), ("n_counters", ctypes.c_int32),
        ("max_instr_per_sm", ctypes.c_int32), ("bytes_min_sm", ctypes.c_int64),
        ("bytes_max_sm", ctypes.c_int64), ("deadlock_free", ctypes.c_int32),
        ("coverage_ok", ctypes.c_int32), ("targets_ok", ctypes.c_int32),
        ("attn_slices", ctypes.c_int32), ("ring_pages", ctypes.c_int32),
        ("smem_bytes", ctypes.c_int32),
    ]


# exported entry points and their signatures (kept in step with include/mk.h)
_SIGS = {
    "mk_create": (ctypes.c_int, [ctypes.POINTER(MkConfig), ctypes.POINTER(MkWeights),
                                 ctypes.POINTER(MkOptions), ctypes.POINTER(ctypes.c_void_p)]),
    "mk_decode_step": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                      ctypes.POINTER(ctypes.c_int32), ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_void_p]),
    "mk_decode_steps": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p,
                                       ctypes.POINTER(ctypes.c_int32), ctypes.c_void_p,
                                       ctypes.c_void_p, ctypes.c_void_p]),
    "mk_decode_step_host": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32,
                                           ctypes.POINTER(ctypes.c_int32),
                                           ctypes.POINTER(ctypes.c_int32), ctypes.c_void_p,
                                           ctypes.POINTER(ctypes.c_int32), ctypes.c_void_p]),
    "mk_prefill": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32),
                                  ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p,
                                  ctypes.POINTER(ctypes.c_int32), ctypes.c_void_p]),
    "mk_sync": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "mk_get_error": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_char_p, ctypes.c_int32]),
    "mk_clear_error": (ctypes.c_int, [ctypes.c_void_p]),
    "mk_destroy": (ctypes.c_int, [ctypes.c_void_p]),
    "mk_plan_check": (ctypes.c_int, [ctypes.POINTER(MkConfig), ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                     ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                     ctypes.POINTER(MkPlanReport)]),
    "mk_rope_inv_freq": (ctypes.c_int, [ctypes.POINTER(MkConfig), ctypes.POINTER(ctypes.c_double),
                                        ctypes.c_int32]),
    "mk_profile_read": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                       ctypes.POINTER(ctypes.c_int32),
                                       ctypes.POINTER(ctypes.c_int32)]),
    "mk_greedy_head_noalloc": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                                              ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                              ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                                              ctypes.c_void_p]),
    "mk_matvec_engine": (ctypes.c_int, [ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                                        ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32,
                                        ctypes.c_int32, ctypes.c_void_p]),
    "mk_matvec_engine_status": (ctypes.c_int, [ctypes.c_void_p]),
    "mk_version": (ctypes.c_char_p, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libmk.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise MkError(4, f"{LIB} is missing; build it with "
                             "`python -m persistent_megakernel_02_b200.build`")
        handle = ctypes.CDLL(LIB)
        for name, (res, args) in _SIGS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def version() -> str:
    return lib().mk_version().decode()


def _check(status: int, what: str):
    if status != 0:
        raise MkError(status, what)


_CFG_FIELDS = [f for f, _ in MkConfig._fields_]


def config_struct(cfg: dict) -> MkConfig:
    return MkConfig(**{k: cfg.get(k, 0) if k == "kv_dtype" else cfg[k] for k in _CFG_FIELDS})


def plan_check(cfg: dict, n_sm: int, nb: int, fault: int = 0, dyn_percent: int = 0, region: int = 0,
               tensor_core_units: int = 0) -> dict:
    """Lower ``cfg`` on the host and run the tape simulator (no GPU needed).
    ``region``: 0 the whole step, 1 the decoder layers, 2 the LM head (region cut);
    ``tensor_core_units``: mk_options.tensor_core_units."""
    rep = MkPlanReport()
    c = config_struct(cfg)
    _check(lib().mk_plan_check(ctypes.byref(c), n_sm, nb, fault, dyn_percent, region, tensor_core_units,
                               ctypes.byref(rep)), "mk_plan_check")
    return {f: getattr(rep, f) for f, _ in MkPlanReport._fields_}


def rope_inv_freq(cfg: dict):
    """The RoPE inverse frequencies the library's table is built from (host only)."""
    n = int(cfg["head_dim"]) // 2
    out = (ctypes.c_double * n)()
    c = config_struct(cfg)
    _check(lib().mk_rope_inv_freq(ctypes.byref(c), out, n), "mk_rope_inv_freq")
    return list(out)


def greedy_head_noalloc(hidden, final_norm, lm_head, rms_eps, ids, logits=None, stream=None):
    """Final RMSNorm + LM head + greedy argmax through ``mk_greedy_head_noalloc``.

    For callers that cannot allocate device memory on their call path: the call
    uses only a static scratch array inside the library.  ``hidden`` is a CUDA
    float32 [nb, H] tensor, ``final_norm`` bf16 [H], ``lm_head`` bf16 [V, H],
    ``ids`` int32 with at least nb elements, ``logits`` float32 [nb, V] or None,
    all contiguous and on the current CUDA device.  The C entry point sees raw
    pointers only, so every shape, dtype, layout and device is checked here
    first; a mismatch raises MkError(MK_ERR_INVALID_ARG) before anything is
    launched.  Asynchronous.
    """
    import torch

    def bad(why):
        raise MkError(1, f"mk_greedy_head_noalloc: {why}")

    if hidden.dim() != 2:
        bad("hidden must be a [nb, hidden] tensor")
    nb, H = (int(x) for x in hidden.shape)
    if lm_head.dim() != 2 or int(lm_head.shape[1]) != H:
        bad("lm_head must be [vocab, hidden]")
    V = int(lm_head.shape[0])
    want = [("hidden", hidden, torch.float32, (nb, H)),
            ("final_norm", final_norm, torch.bfloat16, (H,)),
            ("lm_head", lm_head, torch.bfloat16, (V, H))]
    if logits is not None:
        want.append(("logits", logits, torch.float32, (nb, V)))
    for name, t, dtype, shape in want:
        if t.dtype != dtype:
            bad(f"{name} must be {dtype}, got {t.dtype}")
        if tuple(t.shape) != shape:
            bad(f"{name} must have shape {shape}, got {tuple(t.shape)}")
        if not t.is_contiguous():
            bad(f"{name} must be contiguous")
    if ids.dtype != torch.int32 or ids.dim() != 1 or ids.numel() < nb or not ids.is_contiguous():
        bad("ids must be a contiguous int32 vector of at least nb elements")
    tensors = [t for _, t, _, _ in want] + [ids]
    if not all(t.is_cuda for t in tensors):
        bad("every tensor must be on a CUDA device")
    dev = torch.cuda.current_device()
    if any(t.device.index != dev for t in tensors):
        bad(f"every tensor must be on the current CUDA device ({dev})")
    _check(lib().mk_greedy_head_noalloc(hidden.data_ptr(), nb, H, final_norm.data_ptr(),
                                        lm_head.data_ptr(), V, rms_eps,
                                        None if logits is None else logits.data_ptr(),
                                        ids.data_ptr(), _stream_handle(stream)),
           "mk_greedy_head_noalloc")


ENGINES = {"cuda_cores": 0, "tcgen05": 1}


def matvec_engine(engine, W, X, Y, n_sm: int = 0, wait_limit_ms: int = 0, stream=None):
    """Y[b, r] = sum_k W[r, k] * X[b, k] on one engine (``mk_matvec_engine``):
    "cuda_cores" or "tcgen05".  W bf16 [rows, K], X float32 [nb, K], Y float32
    [nb, rows], all CUDA tensors.  Asynchronous; ``matvec_engine_status`` waits."""
    rows, K = W.shape
    nb = X.shape[0]
    _check(lib().mk_matvec_engine(ENGINES[engine], W.data_ptr(), rows, K, X.data_ptr(), nb, Y.data_ptr(),
                                  n_sm, wait_limit_ms, _stream_handle(stream)), "mk_matvec_engine")


def matvec_engine_status(stream=None):
    _check(lib().mk_matvec_engine_status(_stream_handle(stream)), "mk_matvec_engine")


def _i32_array(values):
    vals = [int(v) for v in values]
    return (ctypes.c_int32 * max(1, len(vals)))(*vals)


def _stream_handle(stream):
    if stream is None:
        return None
    return ctypes.c_void_p(getattr(stream, "cuda_stream", stream))


class Megakernel:
    """One decoder handle over caller-owned bf16 CUDA weights.

    ``weights`` is the dict of :func:`synth.make_weights` layout: 'embed',
    'lm_head' (None when tied), 'final_norm' and per-layer lists 'attn_norm',
    'wq', 'wk', 'wv', 'wo', 'mlp_norm', 'w_gate', 'w_up', 'w_down' -- contiguous
    bf16 CUDA tensors.  The handle keeps references to them.  The keyword options
    are mk_options' fields (include/mk.h); ``dyn_percent`` > 0 leaves that share of
    the gate/up, down and LM-head rows to run-time claims; ``prefill_tokenwise`` = 1
    runs prompts token by token through the decode kernel instead of batched;
    ``region_cut`` = 1 runs each decode step as two launches (layers, LM head);
    ``tensor_core_units`` picks the 8-lane matvecs on tcgen05 (0 measured default,
    1 none, 2 LM head, 3 gate/up, 4 both).
    """

    _LAYER = ("attn_norm", "wq", "wk", "wv", "wo", "mlp_norm", "w_gate", "w_up", "w_down")

    def __init__(self, cfg: dict, weights: dict, device: int = 0, wait_limit_ms: int = 1000,
                 n_sm: int = 0, ring_pages: int = 0, debug_fault: int = 0, profile: int = 0,
                 dyn_percent: int = 0, prefill_tokenwise: int = 0, region_cut: int = 0,
                 tensor_core_units: int = 0):
        self.cfg = dict(cfg)
        self._host_io = None
        self._weights = weights
        self._arrays = {}
        for name in self._LAYER:
            ptrs = [t.data_ptr() for t in weights[name]]
            self._arrays[name] = (ctypes.c_void_p * len(ptrs))(*ptrs)
        w = MkWeights(
            embed=weights["embed"].data_ptr(),
            lm_head=None if weights.get("lm_head") is None else weights["lm_head"].data_ptr(),
            final_norm=weights["final_norm"].data_ptr(),
            **{n: ctypes.cast(self._arrays[n], _PP) for n in self._LAYER},
        )
        opt = MkOptions(device=device, wait_limit_ms=wait_limit_ms, n_sm=n_sm,
                        ring_pages=ring_pages, debug_fault=debug_fault, profile=profile,
                        dyn_percent=dyn_percent, prefill_tokenwise=prefill_tokenwise,
                        region_cut=region_cut, tensor_core_units=tensor_core_units)
        self._cfg_struct = config_struct(cfg)
        h = ctypes.c_void_p()
        _check(lib().mk_create(ctypes.byref(self._cfg_struct), ctypes.byref(w), ctypes.byref(opt),
                               ctypes.byref(h)), "mk_create")
        self._h = h

    # -- steps ------------------------------------------------------------
    def decode_step(self, tokens, positions, ids, logits=None, stream=None):
        """Asynchronous step over device tensors (tokens/ids int32 [nb], logits f32 [nb, V])."""
        nb = len(positions)
        _check(lib().mk_decode_step(self._h, nb, tokens.data_ptr(), _i32_array(positions),
                                    None if logits is None else logits.data_ptr(), ids.data_ptr(),
                                    _stream_handle(stream)), "mk_decode_step")

    def decode_steps(self, tokens, positions, n_steps, ids, logits=None, stream=None):
        """n_steps chained greedy steps in one launch; ids int32 [n_steps, nb] (device),
        logits None or float32 [n_steps, nb, V]."""
        nb = len(positions)
        _check(lib().mk_decode_steps(self._h, nb, n_steps, tokens.data_ptr(), _i32_array(positions),
                                     None if logits is None else logits.data_ptr(), ids.data_ptr(),
                                     _stream_handle(stream)), "mk_decode_steps")

    def decode_step_host(self, tokens, positions, want_logits=False, stream=None):
        """Step over host buffers; returns (ids list, logits numpy [nb, V] or None)."""
        nb = len(positions)
        if len(tokens) != nb or not 1 <= nb <= 8:
            raise MkError(1, "mk_decode_step_host: one token and one position per lane, 1..8 lanes")
        io = self._host_io
        if io is None:  # argument buffers reused by every call
            io = self._host_io = tuple((ctypes.c_int32 * 8)() for _ in range(3))
        tk, ps, ids = io
        try:
            tk[:nb] = tokens
            ps[:nb] = positions
        except TypeError:  # e.g. tensors: element by element
            for i in range(nb):
                tk[i] = int(tokens[i])
                ps[i] = int(positions[i])
        lg = None
        if want_logits:
            import numpy as np

            lg = np.empty((nb, self.cfg["vocab"]), dtype=np.float32)
        st = lib().mk_decode_step_host(self._h, nb, tk, ps, None if lg is None else lg.ctypes.data_as(ctypes.c_void_p),
                                       ids, None if stream is None else _stream_handle(stream))
        if st:
            raise MkError(st, "mk_decode_step_host")
        return ids[:nb], lg

    def prefill(self, seq, tokens, start_pos=0, logits_last=None, want_id=True, stream=None):
        """Run the prompt of slot ``seq`` token by token; returns the last greedy id."""
        toks = _i32_array(tokens)
        out = ctypes.c_int32(-1)
        _check(lib().mk_prefill(self._h, seq, toks, len(tokens), start_pos,
                                None if logits_last is None else logits_last.data_ptr(),
                                ctypes.byref(out) if want_id else None, _stream_handle(stream)),
               "mk_prefill")
        return out.value if want_id else None

    def profile_records(self):
        """Per-instruction profile records: int64 array [n_sm, stride, 32] (see mk_profile_read)."""
        import numpy as np

        n_sm, stride = ctypes.c_int32(), ctypes.c_int32()
        lib().mk_profile_read(self._h, None, 0, ctypes.byref(n_sm), ctypes.byref(stride))
        out = np.zeros((n_sm.value, stride.value, 32), dtype=np.int64)
        _check(lib().mk_profile_read(self._h, out.ctypes.data_as(ctypes.c_void_p), out.size,
                                     ctypes.byref(n_sm), ctypes.byref(stride)), "mk_profile_read")
        return out

    def sync(self, stream=None):
        _check(lib().mk_sync(self._h, _stream_handle(stream)), "mk_sync")

    def status(self, stream=None) -> int:
        """mk_sync's status without raising."""
        return lib().mk_sync(self._h, _stream_handle(stream))

    def error_string(self) -> str:
        buf = ctypes.create_string_buffer(256)
        lib().mk_get_error(self._h, buf, 256)
        return buf.value.decode()

    def clear_error(self):
        _check(lib().mk_clear_error(self._h), "mk_clear_error")

    def close(self):
        if getattr(self, "_h", None):
            lib().mk_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
