"""Sparse masked-diffusion sampling on B200 (sm_100a).

Python binding of the C ABI in ``include/smdm.h`` (library ``libsmdm.so`` in this package).
The binding only marshals arguments: torch supplies device memory and streams, every step of
the computation runs in the library's CUDA kernels.  There is no CPU fallback: importing works
anywhere, but creating a model raises if the library is not built or no GPU is present.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsmdm.so")

# --- constants mirrored from smdm.h ----------------------------------------------------------
SMDM_OK, SMDM_EINVAL, SMDM_ESHAPE, SMDM_ENOMEM, SMDM_ECUDA, SMDM_ESTATE, SMDM_ETIMEOUT, \
    SMDM_EDEVICE = range(8)
SMDM_F32, SMDM_BF16 = 0, 1
SMDM_POLICY_ALL, SMDM_POLICY_TOPN = 0, 1
SMDM_MODE_SPARSE, SMDM_MODE_DENSE = 0, 1
SMDM_TYPE_PROMPT, SMDM_TYPE_CLEAN, SMDM_TYPE_MASK, SMDM_TYPE_REG = range(4)
SMDM_PLAN_ORDER, SMDM_PLAN_SEMIAR = 0, 1
SMDM_MAX_BATCH = 8
SMDM_REG_LEN = -1      # n_reg of the length-token variant (one [LEN] row, no registers)
SMDM_SW_CACHE_PROMPT, SMDM_SW_CACHE_RES, SMDM_SW_TRUNCATE, SMDM_SW_ALL = 1, 2, 4, 7

STATUS_NAMES = {0: "SMDM_OK", 1: "SMDM_EINVAL", 2: "SMDM_ESHAPE", 3: "SMDM_ENOMEM",
                4: "SMDM_ECUDA", 5: "SMDM_ESTATE", 6: "SMDM_ETIMEOUT", 7: "SMDM_EDEVICE"}

EXPORTED = ["smdm_workspace_bytes", "smdm_create", "smdm_destroy", "smdm_last_error",
            "smdm_prefill", "smdm_prefill_given", "smdm_step", "smdm_step_switched",
            "smdm_dense_step", "smdm_generate",
            "smdm_forward_stepcausal", "smdm_debug_mask", "smdm_debug_rows",
            "smdm_context_length", "smdm_device_status", "smdm_profile_begin",
            "smdm_profile_end", "smdm_forward_stepcausal_noalloc"]

K_CLASSES = ["pack", "norm", "gemm_qkv", "attn", "gemm_o", "gemm_gateup", "gemm_down",
             "gemm_lmhead", "unmask", "other"]


class SmdmError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class smdm_config(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("d_model", ctypes.c_int), ("n_heads", ctypes.c_int),
                ("d_head", ctypes.c_int), ("d_ffn", ctypes.c_int), ("vocab", ctypes.c_int),
                ("n_reg", ctypes.c_int), ("dtype", ctypes.c_int), ("rope_theta", ctypes.c_float),
                ("rms_eps", ctypes.c_float), ("max_batch", ctypes.c_int),
                ("max_len", ctypes.c_int), ("max_step_rows", ctypes.c_int),
                ("max_rows", ctypes.c_int)]


_PP = ctypes.POINTER(ctypes.c_void_p)


class smdm_weights(ctypes.Structure):
    _fields_ = [("emb", ctypes.c_void_p), ("final_norm", ctypes.c_void_p),
                ("lm_head", ctypes.c_void_p), ("attn_norm", _PP), ("w_qkv", _PP), ("w_o", _PP),
                ("mlp_norm", _PP), ("w_gate", _PP), ("w_up", _PP), ("w_down", _PP)]


class smdm_step_desc(ctypes.Structure):
    _fields_ = [("seq", ctypes.c_int), ("d_query_pos", ctypes.c_void_p),
                ("n_query", ctypes.c_int), ("block_lo", ctypes.c_int), ("block_hi", ctypes.c_int),
                ("policy", ctypes.c_int), ("n_commit", ctypes.c_int)]


class smdm_plan(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("n_steps", ctypes.c_int),
                ("h_n_per_step", ctypes.POINTER(ctypes.c_int32)), ("d_order", ctypes.c_void_p),
                ("block", ctypes.c_int), ("steps_per_block", ctypes.c_int),
                ("commit", ctypes.c_int), ("h_block_order", ctypes.POINTER(ctypes.c_int32))]


class smdm_profile(ctypes.Structure):
    _fields_ = [("launches", ctypes.c_ulonglong), ("class_launches", ctypes.c_ulonglong * 10),
                ("class_ms", ctypes.c_double * 10)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libsmdm.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m masked_discrete_diffusion_sparse_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, st = ctypes.c_void_p, ctypes.c_int, ctypes.c_int
    L.smdm_workspace_bytes.argtypes = [ctypes.POINTER(smdm_config)]
    L.smdm_workspace_bytes.restype = ctypes.c_size_t
    L.smdm_create.argtypes = [ctypes.POINTER(smdm_config), ctypes.POINTER(smdm_weights), vp,
                              ctypes.c_size_t, ctypes.POINTER(vp)]
    L.smdm_create.restype = st
    L.smdm_destroy.argtypes = [vp]
    L.smdm_destroy.restype = None
    L.smdm_last_error.argtypes = [vp]
    L.smdm_last_error.restype = ctypes.c_char_p
    L.smdm_prefill.argtypes = [vp, i32, vp, i32, i32, vp, vp]
    L.smdm_prefill.restype = st
    L.smdm_prefill_given.argtypes = [vp, i32, vp, i32, i32, vp, vp, i32, vp, vp]
    L.smdm_prefill_given.restype = st
    L.smdm_step.argtypes = [vp, i32, ctypes.POINTER(smdm_step_desc), vp, vp, vp, vp]
    L.smdm_step.restype = st
    L.smdm_step_switched.argtypes = [vp, ctypes.POINTER(smdm_step_desc), i32, vp, vp, vp, vp]
    L.smdm_step_switched.restype = st
    L.smdm_dense_step.argtypes = [vp, ctypes.POINTER(smdm_step_desc), vp, vp, vp, vp]
    L.smdm_dense_step.restype = st
    L.smdm_generate.argtypes = [vp, i32, vp, i32, i32, ctypes.POINTER(smdm_plan), i32, vp, vp]
    L.smdm_generate.restype = st
    L.smdm_forward_stepcausal.argtypes = [vp, vp, vp, vp, vp, i32, vp, i32, vp, vp]
    L.smdm_forward_stepcausal.restype = st
    L.smdm_debug_mask.argtypes = [vp, vp, vp, i32, vp, vp]
    L.smdm_debug_mask.restype = st
    L.smdm_debug_rows.argtypes = [vp, vp, vp, vp, vp, ctypes.POINTER(ctypes.c_int), vp]
    L.smdm_debug_rows.restype = st
    L.smdm_context_length.argtypes = [vp, i32]
    L.smdm_context_length.restype = ctypes.c_int
    L.smdm_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint), vp]
    L.smdm_device_status.restype = st
    L.smdm_profile_begin.argtypes = [vp, i32]
    L.smdm_profile_begin.restype = st
    L.smdm_profile_end.argtypes = [vp, ctypes.POINTER(smdm_profile), vp]
    L.smdm_profile_end.restype = st
    L.smdm_forward_stepcausal_noalloc.argtypes = [ctypes.POINTER(smdm_config),
                                                  ctypes.POINTER(smdm_weights), vp, vp, vp, vp,
                                                  i32, vp, i32, vp, vp]
    L.smdm_forward_stepcausal_noalloc.restype = st
    _lib = L
    return L


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _i32(t: torch.Tensor) -> torch.Tensor:
    if t.dtype != torch.int32:
        raise ValueError("expected an int32 tensor")
    return t


class Model:
    """A handle plus the device memory it borrows.

    weights: dict with 'emb', 'final_norm', 'lm_head' and per-layer lists 'attn_norm', 'w_qkv',
    'w_o', 'mlp_norm', 'w_gate', 'w_up', 'w_down' (torch CUDA tensors in the model dtype, linear
    weights [out][in]).  Methods mirror the C entry points of the same name.
    """

    def __init__(self, cfg: smdm_config, weights: dict, device: str = "cuda"):
        L = lib()
        if not torch.cuda.is_available():
            raise RuntimeError("the sparse sampler needs a CUDA device (no CPU fallback)")
        self.cfg = cfg
        self.weights = weights
        self._layer_arrays = {}
        arr = {}
        for k in ("attn_norm", "w_qkv", "w_o", "mlp_norm", "w_gate", "w_up", "w_down"):
            ts = weights[k]
            a = (ctypes.c_void_p * cfg.n_layers)(*[t.data_ptr() for t in ts])
            self._layer_arrays[k] = a
            arr[k] = ctypes.cast(a, _PP)
        self._w = smdm_weights(weights["emb"].data_ptr(), weights["final_norm"].data_ptr(),
                               weights["lm_head"].data_ptr(), arr["attn_norm"], arr["w_qkv"],
                               arr["w_o"], arr["mlp_norm"], arr["w_gate"], arr["w_up"],
                               arr["w_down"])
        nbytes = L.smdm_workspace_bytes(ctypes.byref(cfg))
        if nbytes == 0:
            raise SmdmError(SMDM_ESHAPE, "invalid configuration")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        torch.cuda.synchronize()
        h = ctypes.c_void_p()
        s = L.smdm_create(ctypes.byref(cfg), ctypes.byref(self._w),
                          ctypes.c_void_p(self.workspace.data_ptr()), nbytes, ctypes.byref(h))
        if s != SMDM_OK:
            raise SmdmError(s, "smdm_create failed")
        self.h = h

    def close(self):
        if getattr(self, "h", None):
            lib().smdm_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, s: int):
        if s != SMDM_OK:
            raise SmdmError(s, lib().smdm_last_error(self.h).decode())

    # -- entry points -------------------------------------------------------------------------
    def smdm_prefill(self, seq: int, prompt: torch.Tensor, gen_len: int, grid: torch.Tensor,
                     stream=None):
        self._check(lib().smdm_prefill(self.h, seq, _ptr(_i32(prompt)) if prompt.numel() else None,
                                       prompt.numel(), gen_len, _ptr(_i32(grid)), _stream(stream)))

    def smdm_prefill_given(self, seq: int, prompt: torch.Tensor, gen_len: int,
                           given_pos: torch.Tensor, given_tok: torch.Tensor, grid: torch.Tensor,
                           stream=None):
        """Prefill with given generation tokens (bidirectional tasks): 1-based absolute
        positions and their token ids, device int32 tensors of equal length."""
        if given_pos.numel() != given_tok.numel():
            raise ValueError("given_pos and given_tok differ in length")
        n = given_pos.numel()
        self._check(lib().smdm_prefill_given(
            self.h, seq, _ptr(_i32(prompt)) if prompt.numel() else None, prompt.numel(), gen_len,
            _ptr(_i32(given_pos)) if n else None, _ptr(_i32(given_tok)) if n else None, n,
            _ptr(_i32(grid)), _stream(stream)))

    def smdm_step(self, descs: Sequence[dict], logits: Optional[torch.Tensor] = None,
                  tok: Optional[torch.Tensor] = None, conf: Optional[torch.Tensor] = None,
                  stream=None):
        """descs: dicts with seq, query_pos (int32 CUDA tensor or None), n_query, block_lo,
        block_hi, policy, n_commit."""
        arr = (smdm_step_desc * len(descs))()
        for i, d in enumerate(descs):
            qp = d.get("query_pos")
            arr[i] = smdm_step_desc(d["seq"], _ptr(_i32(qp)) if qp is not None else None,
                                    d["n_query"], d.get("block_lo", 0), d.get("block_hi", 0),
                                    d.get("policy", SMDM_POLICY_ALL), d.get("n_commit", 0))
        self._check(lib().smdm_step(self.h, len(descs), arr, _ptr(logits), _ptr(tok), _ptr(conf),
                                    _stream(stream)))

    def smdm_step_switched(self, desc: dict, switches: int, logits=None, tok=None, conf=None,
                           stream=None):
        """One step of one sequence with the Table-6 speed switches (SMDM_SW_* bits); desc as
        in smdm_step, with query_pos required."""
        qp = desc["query_pos"]
        d = smdm_step_desc(desc["seq"], _ptr(_i32(qp)), desc["n_query"], 0, 0,
                           desc.get("policy", SMDM_POLICY_ALL), desc.get("n_commit", 0))
        self._check(lib().smdm_step_switched(self.h, ctypes.byref(d), switches, _ptr(logits),
                                             _ptr(tok), _ptr(conf), _stream(stream)))

    def smdm_dense_step(self, desc: dict, logits=None, tok=None, conf=None, stream=None):
        qp = desc.get("query_pos")
        d = smdm_step_desc(desc["seq"], _ptr(_i32(qp)) if qp is not None else None,
                           desc["n_query"], desc.get("block_lo", 0), desc.get("block_hi", 0),
                           desc.get("policy", SMDM_POLICY_ALL), desc.get("n_commit", 0))
        self._check(lib().smdm_dense_step(self.h, ctypes.byref(d), _ptr(logits), _ptr(tok),
                                          _ptr(conf), _stream(stream)))

    def smdm_generate(self, prompts: torch.Tensor, gen_len: int, plans: Sequence[dict],
                      grids: torch.Tensor, mode: int = SMDM_MODE_SPARSE, stream=None):
        """plans: dicts with kind, n_steps, n_per_step (host int list), order (int32 CUDA
        tensor), block, steps_per_block, commit, block_order (host int list, optional)."""
        B = len(plans)
        arr = (smdm_plan * B)()
        keep = []
        for i, p in enumerate(plans):
            nps = p.get("n_per_step")
            h_n = None
            if nps is not None:
                h_n = (ctypes.c_int32 * len(nps))(*[int(v) for v in nps])
                keep.append(h_n)
            bo = p.get("block_order")
            h_bo = None
            if bo is not None:
                h_bo = (ctypes.c_int32 * len(bo))(*[int(v) for v in bo])
                keep.append(h_bo)
            order = p.get("order")
            arr[i] = smdm_plan(p["kind"], p["n_steps"],
                               ctypes.cast(h_n, ctypes.POINTER(ctypes.c_int32)) if h_n else None,
                               _ptr(_i32(order)) if order is not None else None,
                               p.get("block", 0), p.get("steps_per_block", 0), p.get("commit", 0),
                               ctypes.cast(h_bo, ctypes.POINTER(ctypes.c_int32)) if h_bo else None)
        P = prompts.shape[-1] if prompts.numel() else 0
        self._check(lib().smdm_generate(self.h, B, _ptr(_i32(prompts)) if P else None, P, gen_len,
                                        arr, mode, _ptr(_i32(grids)), _stream(stream)))

    def smdm_forward_stepcausal(self, ids, pos, types, labels, logit_rows, logits, stream=None):
        self._check(lib().smdm_forward_stepcausal(
            self.h, _ptr(_i32(ids)), _ptr(_i32(pos)), _ptr(_i32(types)), _ptr(_i32(labels)),
            ids.numel(), _ptr(_i32(logit_rows)), logit_rows.numel(), _ptr(logits),
            _stream(stream)))

    def smdm_debug_mask(self, types, labels, bitmap, stream=None):
        self._check(lib().smdm_debug_mask(self.h, _ptr(_i32(types)), _ptr(_i32(labels)),
                                          types.numel(), _ptr(bitmap), _stream(stream)))

    def smdm_debug_rows(self, ids=None, pos=None, types=None, labels=None, stream=None) -> int:
        n = ctypes.c_int(0)
        self._check(lib().smdm_debug_rows(self.h, _ptr(ids), _ptr(pos), _ptr(types), _ptr(labels),
                                          ctypes.byref(n), _stream(stream)))
        return n.value

    def smdm_context_length(self, seq: int) -> int:
        return lib().smdm_context_length(self.h, seq)

    def smdm_profile_begin(self, timed: bool = False):
        self._check(lib().smdm_profile_begin(self.h, 1 if timed else 0))

    def smdm_profile_end(self, stream=None) -> dict:
        p = smdm_profile()
        self._check(lib().smdm_profile_end(self.h, ctypes.byref(p), _stream(stream)))
        return {"launches": int(p.launches),
                "class_launches": {K_CLASSES[i]: int(p.class_launches[i]) for i in range(10)},
                "class_ms": {K_CLASSES[i]: float(p.class_ms[i]) for i in range(10)}}

    def smdm_device_status(self, stream=None) -> int:
        bits = ctypes.c_uint(0)
        self._check(lib().smdm_device_status(self.h, ctypes.byref(bits), _stream(stream)))
        return bits.value


def smdm_forward_stepcausal_noalloc(cfg: smdm_config, weights: dict, ids, pos, types, labels,
                                    logit_rows, logits, stream=None):
    """Training-form forward without a handle and without any device allocation.

    For callers that may not allocate device memory at the point of the call (a frozen
    allocator, a plug-in handed only pointers by its host program): all scratch lives in a
    16 MiB array built into the library.  Same arguments and result as
    Model.smdm_forward_stepcausal, plus the config and the weights dict.  Shapes whose scratch
    does not fit raise SmdmError(SMDM_ESHAPE).  Calls share that array: do not overlap them on
    the GPU.  Make the first call on a device outside CUDA-graph capture (it looks up the
    array's device address).
    """
    keep = []
    arr = {}
    for k in ("attn_norm", "w_qkv", "w_o", "mlp_norm", "w_gate", "w_up", "w_down"):
        a = (ctypes.c_void_p * cfg.n_layers)(*[t.data_ptr() for t in weights[k]])
        keep.append(a)
        arr[k] = ctypes.cast(a, _PP)
    w = smdm_weights(weights["emb"].data_ptr(), weights["final_norm"].data_ptr(),
                     weights["lm_head"].data_ptr(), arr["attn_norm"], arr["w_qkv"], arr["w_o"],
                     arr["mlp_norm"], arr["w_gate"], arr["w_up"], arr["w_down"])
    s = lib().smdm_forward_stepcausal_noalloc(
        ctypes.byref(cfg), ctypes.byref(w), _ptr(_i32(ids)), _ptr(_i32(pos)), _ptr(_i32(types)),
        _ptr(_i32(labels)), ids.numel(), _ptr(_i32(logit_rows)), logit_rows.numel(),
        _ptr(logits), _stream(stream))
    if s != SMDM_OK:
        raise SmdmError(s, "smdm_forward_stepcausal_noalloc failed")


def make_config(n_layers, d_model, n_heads, d_head, d_ffn, vocab, n_reg=64, dtype=SMDM_BF16,
                rope_theta=10000.0, rms_eps=1e-6, max_batch=1, max_len=1, max_step_rows=1,
                max_rows=1) -> smdm_config:
    return smdm_config(n_layers, d_model, n_heads, d_head, d_ffn, vocab, n_reg, dtype, rope_theta,
                       rms_eps, max_batch, max_len, max_step_rows, max_rows)
