"""Thin Python binding of the C ABI in ``include/specopd.h``.

Argument marshalling only: every step of the hot path runs in the CUDA
kernels of ``libspecopd.so``.  Tensors are torch CUDA tensors (PyTorch
supplies device memory and streams); each call passes ``data_ptr()`` and the
current stream's handle and raises ``SpecopdError`` on a non-OK status.
There is no fallback: if the library is missing or no sm_100 device is
present, calls fail loudly.
"""

from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libspecopd.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "specopd.h")

F32, BF16 = 0, 1
DEV_ANCHOR_RANGE, DEV_ROW_RANGE, DEV_ALL_NEG_INF, DEV_TIMEOUT, DEV_LAYOUT = 0x1, 0x2, 0x4, 0x8, 0x10

_STATUS = {0: "SPECOPD_OK", 1: "SPECOPD_ERR_INVALID_ARG", 2: "SPECOPD_ERR_UNSUPPORTED",
           3: "SPECOPD_ERR_WORKSPACE", 4: "SPECOPD_ERR_CUDA", 5: "SPECOPD_ERR_TIMEOUT",
           6: "SPECOPD_ERR_NO_DEVICE"}


class SpecopdError(RuntimeError):
    def __init__(self, status, what=""):
        self.status = status
        super().__init__(f"{what}: {_STATUS.get(status, status)}")


class AttnDesc(ctypes.Structure):
    _fields_ = [("S", ctypes.c_int), ("B", ctypes.c_int), ("W", ctypes.c_int),
                ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("D", ctypes.c_int),
                ("dtype", ctypes.c_int), ("rope_base", ctypes.c_float),
                ("softmax_scale", ctypes.c_float)]


class RopeDesc(ctypes.Structure):
    _fields_ = [("D", ctypes.c_int), ("dtype", ctypes.c_int), ("rope_base", ctypes.c_float)]


class TVDesc(ctypes.Structure):
    _fields_ = [("nbranch", ctypes.c_int), ("W", ctypes.c_int), ("V", ctypes.c_int),
                ("rows_target", ctypes.c_int), ("logit_dtype", ctypes.c_int),
                ("grad_dtype", ctypes.c_int), ("compute_grad", ctypes.c_int),
                ("norm_count", ctypes.c_int64)]


class LmheadTVDesc(ctypes.Structure):
    _fields_ = [("nbranch", ctypes.c_int), ("W", ctypes.c_int), ("V", ctypes.c_int),
                ("d_model", ctypes.c_int), ("rows_target", ctypes.c_int),
                ("grad_dtype", ctypes.c_int), ("compute_grad", ctypes.c_int),
                ("norm_count", ctypes.c_int64)]


_lib = None


def load(path: str = LIB_PATH):
    """Load libspecopd.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python tree_attention_specopd_b200/build.py` (needs nvcc)")
    lib = ctypes.CDLL(path)
    vp, i32p, f32p, f64p = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
    cint, csize = ctypes.c_int, ctypes.c_size_t
    lib.specopd_status_string.restype = ctypes.c_char_p
    lib.specopd_status_string.argtypes = [cint]
    lib.specopd_version.restype = cint
    lib.specopd_get_device_status.restype = cint
    lib.specopd_get_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint32), vp]
    lib.specopd_tree_build.restype = cint
    lib.specopd_tree_build.argtypes = [cint, ctypes.POINTER(ctypes.c_int32), i32p, cint, cint,
                                       i32p, i32p, i32p, vp]
    lib.specopd_rope_apply.restype = cint
    lib.specopd_rope_apply.argtypes = [ctypes.POINTER(RopeDesc), vp, i32p, cint, cint, vp]
    lib.specopd_tree_attn_workspace_size.restype = csize
    lib.specopd_tree_attn_workspace_size.argtypes = [ctypes.POINTER(AttnDesc),
                                                     ctypes.POINTER(ctypes.c_int32)]
    lib.specopd_tree_attn.restype = cint
    lib.specopd_tree_attn.argtypes = [ctypes.POINTER(AttnDesc), vp, vp, vp, vp, vp, i32p,
                                      ctypes.POINTER(ctypes.c_int32), i32p, i32p, vp, f32p,
                                      vp, csize, vp]
    lib.specopd_trunk_prefill_workspace_size.restype = csize
    lib.specopd_trunk_prefill_workspace_size.argtypes = [ctypes.POINTER(AttnDesc),
                                                         ctypes.POINTER(ctypes.c_int32)]
    lib.specopd_trunk_prefill.restype = cint
    lib.specopd_trunk_prefill.argtypes = [ctypes.POINTER(AttnDesc), vp, vp, vp, i32p,
                                          ctypes.POINTER(ctypes.c_int32), vp, f32p, vp, csize, vp]
    lib.specopd_e2e_tv_workspace_size.restype = csize
    lib.specopd_e2e_tv_workspace_size.argtypes = [ctypes.POINTER(TVDesc)]
    lib.specopd_e2e_tv.restype = cint
    lib.specopd_e2e_tv.argtypes = [ctypes.POINTER(TVDesc), vp, i32p, vp, f32p, f32p, f32p,
                                   f64p, vp, vp, csize, vp]
    lib.specopd_e2e_tv_noalloc.restype = cint
    lib.specopd_e2e_tv_noalloc.argtypes = [ctypes.POINTER(TVDesc), vp, i32p, vp, f32p, f32p,
                                           f32p, f64p, vp, vp]
    lib.specopd_e2e_tv_lmhead_workspace_size.restype = csize
    lib.specopd_e2e_tv_lmhead_workspace_size.argtypes = [ctypes.POINTER(LmheadTVDesc)]
    lib.specopd_e2e_tv_lmhead.restype = cint
    lib.specopd_e2e_tv_lmhead.argtypes = [ctypes.POINTER(LmheadTVDesc), vp, i32p, vp, vp, vp,
                                          f32p, f32p, f32p, f64p, vp, vp, csize, vp]
    lib.specopd_e2e_tv_finalize.restype = cint
    lib.specopd_e2e_tv_finalize.argtypes = [f64p, ctypes.c_int64, f32p, f64p, vp]
    lib.specopd_debug_fault_injection.restype = cint
    lib.specopd_debug_fault_injection.argtypes = [ctypes.c_int64, ctypes.c_uint64]
    _lib = lib
    return lib


def header_functions(path: str = HEADER) -> list[str]:
    """Names of the functions include/specopd.h declares."""
    txt = open(path).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(specopd_[a-z0-9_]+)\s*\(", txt)))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(st, what):
    if st != 0:
        raise SpecopdError(st, what)


def _cu_host(cu_trunk):
    vals = [int(x) for x in (cu_trunk.tolist() if hasattr(cu_trunk, "tolist") else cu_trunk)]
    return (ctypes.c_int32 * len(vals))(*vals), vals


def _dtype_code(t):
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def specopd_get_device_status(stream=None) -> int:
    v = ctypes.c_uint32(0)
    _check(load().specopd_get_device_status(ctypes.byref(v), _stream(stream)), "get_device_status")
    return int(v.value)


def specopd_tree_build(cu_trunk, anchors, B, W, parent=None, sem_pos=None, score_row=None,
                       stream=None):
    """Returns (parent, sem_pos, score_row) int32 CUDA tensors."""
    cu_arr, cu = _cu_host(cu_trunk)
    S = len(cu) - 1
    T_tot, R, N = cu[-1], S * B * (W - 1), S * B * W
    dev = anchors.device
    if parent is None:
        parent = torch.empty(T_tot + R, dtype=torch.int32, device=dev)
    if sem_pos is None:
        sem_pos = torch.empty(T_tot + R, dtype=torch.int32, device=dev)
    if score_row is None:
        score_row = torch.empty(N, dtype=torch.int32, device=dev)
    _check(load().specopd_tree_build(S, cu_arr, _ptr(anchors), B, W, _ptr(parent), _ptr(sem_pos),
                                     _ptr(score_row), _stream(stream)), "tree_build")
    return parent, sem_pos, score_row


def specopd_rope_apply(x, pos, rope_base=10000.0, stream=None):
    """In place: x [n, H, D] rotated at pos [n] (int32)."""
    n, H, D = x.shape
    d = RopeDesc(D, _dtype_code(x), rope_base)
    _check(load().specopd_rope_apply(ctypes.byref(d), _ptr(x), _ptr(pos), n, H, _stream(stream)),
           "rope_apply")
    return x


def attn_desc(S, B, W, Hq, Hkv, D, dtype, rope_base=10000.0, softmax_scale=0.0):
    code = dtype if isinstance(dtype, int) else (BF16 if dtype in ("bf16", torch.bfloat16) else F32)
    return AttnDesc(S, B, W, Hq, Hkv, D, code, rope_base, softmax_scale)


def specopd_tree_attn_workspace_size(desc, cu_trunk) -> int:
    cu_arr, _ = _cu_host(cu_trunk)
    return int(load().specopd_tree_attn_workspace_size(ctypes.byref(desc), cu_arr))


def specopd_tree_attn(desc, q_br, k_br, v_br, k_tr, v_tr, cu_trunk_dev, cu_trunk_host, anchors,
                      sem_pos, out=None, lse=None, workspace=None, stream=None):
    cu_arr, _ = _cu_host(cu_trunk_host)
    if out is None:
        out = torch.empty_like(q_br)
    if workspace is None:
        n = specopd_tree_attn_workspace_size(desc, cu_trunk_host)
        workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=q_br.device)
    _check(load().specopd_tree_attn(ctypes.byref(desc), _ptr(q_br), _ptr(k_br), _ptr(v_br),
                                    _ptr(k_tr), _ptr(v_tr), _ptr(cu_trunk_dev), cu_arr,
                                    _ptr(anchors), _ptr(sem_pos), _ptr(out), _ptr(lse),
                                    _ptr(workspace), workspace.numel(), _stream(stream)),
           "tree_attn")
    return out


def specopd_trunk_prefill_workspace_size(desc, cu_trunk) -> int:
    cu_arr, _ = _cu_host(cu_trunk)
    return int(load().specopd_trunk_prefill_workspace_size(ctypes.byref(desc), cu_arr))


def specopd_trunk_prefill(desc, q_tr, k_tr, v_tr, cu_trunk_dev, cu_trunk_host, out=None, lse=None,
                          workspace=None, stream=None):
    """Causal attention of every trunk row over its own sequence; k_tr is
    rotated in place (it becomes the K cache).  Returns out [T_tot, Hq, D]."""
    cu_arr, _ = _cu_host(cu_trunk_host)
    if out is None:
        out = torch.empty_like(q_tr)
    if workspace is None:
        n = specopd_trunk_prefill_workspace_size(desc, cu_trunk_host)
        workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=q_tr.device)
    _check(load().specopd_trunk_prefill(ctypes.byref(desc), _ptr(q_tr), _ptr(k_tr), _ptr(v_tr),
                                        _ptr(cu_trunk_dev), cu_arr, _ptr(out), _ptr(lse),
                                        _ptr(workspace), workspace.numel(), _stream(stream)),
           "trunk_prefill")
    return out


def tv_desc(nbranch, W, V, rows_target, logit_dtype, grad_dtype="f32", compute_grad=True,
            norm_count=0):
    def code(d):
        return d if isinstance(d, int) else (BF16 if d in ("bf16", torch.bfloat16) else F32)
    return TVDesc(nbranch, W, V, rows_target, code(logit_dtype), code(grad_dtype),
                  1 if compute_grad else 0, int(norm_count))


def specopd_e2e_tv_workspace_size(desc) -> int:
    return int(load().specopd_e2e_tv_workspace_size(ctypes.byref(desc)))


def specopd_e2e_tv(desc, z_target, target_row, z_draft, a=None, prefix=None, loss=None,
                   numer=None, grad=None, workspace=None, stream=None):
    """Returns dict(a, prefix, loss, numer, grad)."""
    dev = z_draft.device
    N = desc.nbranch * desc.W
    if a is None:
        a = torch.empty(N, dtype=torch.float32, device=dev)
    if prefix is None:
        prefix = torch.empty(N, dtype=torch.float32, device=dev)
    if loss is None:
        loss = torch.empty(1, dtype=torch.float32, device=dev)
    if numer is None:
        numer = torch.empty(1, dtype=torch.float64, device=dev)
    if grad is None and desc.compute_grad:
        gdt = torch.bfloat16 if desc.grad_dtype == BF16 else torch.float32
        grad = torch.empty((N, desc.V), dtype=gdt, device=dev)
    if workspace is None:
        workspace = torch.empty(max(specopd_e2e_tv_workspace_size(desc), 256), dtype=torch.uint8,
                                device=dev)
    _check(load().specopd_e2e_tv(ctypes.byref(desc), _ptr(z_target), _ptr(target_row),
                                 _ptr(z_draft), _ptr(a), _ptr(prefix), _ptr(loss), _ptr(numer),
                                 _ptr(grad), _ptr(workspace), workspace.numel(), _stream(stream)),
           "e2e_tv")
    return {"a": a, "prefix": prefix, "loss": loss, "numer": numer, "grad": grad}


def lmhead_tv_desc(nbranch, W, V, d_model, rows_target, grad_dtype="f32", compute_grad=True,
                   norm_count=0):
    g = grad_dtype if isinstance(grad_dtype, int) else (
        BF16 if grad_dtype in ("bf16", torch.bfloat16) else F32)
    return LmheadTVDesc(nbranch, W, V, d_model, rows_target, g, 1 if compute_grad else 0,
                        int(norm_count))


def specopd_e2e_tv_lmhead_workspace_size(desc) -> int:
    return int(load().specopd_e2e_tv_lmhead_workspace_size(ctypes.byref(desc)))


def specopd_e2e_tv_lmhead(desc, h_target, target_row, w_target, h_draft, w_draft, a=None,
                          prefix=None, loss=None, numer=None, grad=None, workspace=None,
                          stream=None):
    """E2E-TV from bf16 hidden rows and LM heads.  Returns dict(a, prefix,
    loss, numer, grad)."""
    dev = h_draft.device
    N = desc.nbranch * desc.W
    if a is None:
        a = torch.empty(N, dtype=torch.float32, device=dev)
    if prefix is None:
        prefix = torch.empty(N, dtype=torch.float32, device=dev)
    if loss is None:
        loss = torch.empty(1, dtype=torch.float32, device=dev)
    if numer is None:
        numer = torch.empty(1, dtype=torch.float64, device=dev)
    if grad is None and desc.compute_grad:
        gdt = torch.bfloat16 if desc.grad_dtype == BF16 else torch.float32
        grad = torch.empty((N, desc.V), dtype=gdt, device=dev)
    if workspace is None:
        workspace = torch.empty(max(specopd_e2e_tv_lmhead_workspace_size(desc), 256),
                                dtype=torch.uint8, device=dev)
    _check(load().specopd_e2e_tv_lmhead(ctypes.byref(desc), _ptr(h_target), _ptr(target_row),
                                        _ptr(w_target), _ptr(h_draft), _ptr(w_draft), _ptr(a),
                                        _ptr(prefix), _ptr(loss), _ptr(numer), _ptr(grad),
                                        _ptr(workspace), workspace.numel(), _stream(stream)),
           "e2e_tv_lmhead")
    return {"a": a, "prefix": prefix, "loss": loss, "numer": numer, "grad": grad}


def specopd_e2e_tv_finalize(numer_sum, norm_count, loss=None, loss64=None, stream=None):
    """loss = 1 - numer_sum / norm_count on the device (numer_sum: the fp64
    sum over ranks of specopd_e2e_tv's numer).  Returns the fp32 loss tensor."""
    if loss is None:
        loss = torch.empty(1, dtype=torch.float32, device=numer_sum.device)
    _check(load().specopd_e2e_tv_finalize(_ptr(numer_sum), int(norm_count), _ptr(loss),
                                          _ptr(loss64), _stream(stream)), "e2e_tv_finalize")
    return loss


def specopd_debug_fault_injection(withhold_position=-1, branch_wait_limit_ns=0):
    """Testing hook: make the E2E-TV scorer of one supervised position skip
    publishing its overlap, and shorten the branch waits that then run out
    (see include/specopd.h).  (-1, 0) turns it off."""
    _check(load().specopd_debug_fault_injection(int(withhold_position), int(branch_wait_limit_ns)),
           "debug_fault_injection")


E2E_TV_STATIC_SCRATCH_BYTES = 8 << 20


def specopd_e2e_tv_noalloc(desc, z_target, target_row, z_draft, a, prefix, loss, numer=None,
                           grad=None, stream=None):
    """E2E-TV without a workspace argument, for callers that cannot allocate
    device memory (the library's fixed 8 MiB scratch array is used instead).
    All outputs are caller-provided; calls that overlap on the GPU race on the
    shared scratch and must be serialised."""
    _check(load().specopd_e2e_tv_noalloc(ctypes.byref(desc), _ptr(z_target), _ptr(target_row),
                                         _ptr(z_draft), _ptr(a), _ptr(prefix), _ptr(loss),
                                         _ptr(numer), _ptr(grad), _stream(stream)),
           "e2e_tv_noalloc")
    return {"a": a, "prefix": prefix, "loss": loss, "numer": numer, "grad": grad}
