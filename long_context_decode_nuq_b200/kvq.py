"""Thin ctypes binding of libkvq.so (argument marshalling only).

Every function here forwards to the C entry point of the same name in
``include/kvq.h``; torch tensors are used only to own device memory and to
name the current CUDA stream.  There is no fallback: if ``libkvq.so`` is
missing or the GPU call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_double, c_int, c_int32, c_size_t, c_void_p

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

KVQ_OK = 0
KVQ_STATUS_OUTLIER_OVERFLOW = 1
KVQ_STATUS_LEN_OVERFLOW = 2
KVQ_STATUS_NOT_EMPTY = 4
KVQ_STATUS_WAIT_TIMEOUT = 8
CHUNK = 64
NOALLOC_SCRATCH_BYTES = 1 << 20  # KVQ_NOALLOC_SCRATCH_BYTES

EXPORTS = (
    "kvq_abi_version", "kvq_strerror", "kvq_validate_cfg", "kvq_layout", "kvq_cache_reset",
    "kvq_quantize_workspace", "kvq_quantize_append", "kvq_decode_qk", "kvq_decode_qk_workspace",
    "kvq_decode_splits",
    "kvq_softmax_merge", "kvq_decode_pv", "kvq_decode_workspace", "kvq_decode_attention",
    "kvq_dequantize", "kvq_fp16_decode_attention", "kvq_fit_workspace", "kvq_fit_codebook",
    "kvq_get_status", "kvq_quantize_append_noalloc", "kvq_decode_partial", "kvq_merge_partials",
    "kvq_decode_attention_fused", "kvq_decode_fused_workspace",
    "kvq_step_input_bytes", "kvq_step_workspace", "kvq_step_create", "kvq_step_launch",
    "kvq_step_destroy",
)


class KvqError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = load().kvq_strerror(code).decode()
        super().__init__(f"{where}: {msg} ({code})")
        self.code = code


class Cfg(ctypes.Structure):
    _fields_ = [("B", c_int32), ("Hq", c_int32), ("Hkv", c_int32), ("D", c_int32),
                ("bits", c_int32), ("T_max", c_int32), ("out_cap_k", c_int32),
                ("out_cap_v", c_int32), ("outlier_frac", c_double), ("rope_theta", c_double)]


_CACHE_FIELDS = ("kcodes", "vcodes", "kthr", "kparams", "vparams", "kout", "vout", "kchunk",
                 "vchunk", "kcount", "vcount", "len", "status")


class CacheStruct(ctypes.Structure):
    _fields_ = [(f, c_void_p) for f in _CACHE_FIELDS]


class CodebookStruct(ctypes.Structure):
    _fields_ = [("levels", c_void_p), ("bounds", c_void_p)]


class Sizes(ctypes.Structure):
    _fields_ = [(f, c_size_t) for f in _CACHE_FIELDS]


class StepDesc(ctypes.Structure):
    _fields_ = [("layers", c_int32), ("caches", POINTER(CacheStruct)),
                ("cbK", POINTER(CodebookStruct)), ("cbV", POINTER(CodebookStruct)),
                ("n_new", c_int32), ("max_len", c_int32), ("splits", c_int32), ("fused", c_int32),
                ("inputs", c_void_p), ("out", c_void_p), ("workspace", c_void_p),
                ("workspace_bytes", c_size_t)]


_lib = None


def load():
    """Load libkvq.so (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with "
                          "`python -m long_context_decode_nuq_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P = c_void_p
    sig = {
        "kvq_abi_version": ([], c_int),
        "kvq_strerror": ([c_int], ctypes.c_char_p),
        "kvq_validate_cfg": ([POINTER(Cfg)], c_int),
        "kvq_layout": ([POINTER(Cfg), POINTER(Sizes)], c_int),
        "kvq_cache_reset": ([POINTER(Cfg), POINTER(CacheStruct), P], c_int),
        "kvq_quantize_workspace": ([POINTER(Cfg), c_int32, c_int32, POINTER(c_size_t)], c_int),
        "kvq_quantize_append": ([POINTER(Cfg), POINTER(CacheStruct), POINTER(CodebookStruct),
                                 POINTER(CodebookStruct), P, P, c_int32, P, c_int32, P, c_size_t,
                                 P], c_int),
        "kvq_decode_qk": ([POINTER(Cfg), POINTER(CacheStruct), POINTER(CodebookStruct), P, P,
                           c_int32, P, P, c_int32, P, c_size_t, P], c_int),
        "kvq_decode_qk_workspace": ([POINTER(Cfg), c_int32, POINTER(c_size_t)], c_int),
        "kvq_decode_splits": ([POINTER(Cfg), c_int32], c_int),
        "kvq_softmax_merge": ([POINTER(Cfg), P, c_int32, P, P], c_int),
        "kvq_decode_pv": ([POINTER(Cfg), POINTER(CacheStruct), POINTER(CodebookStruct), P, P,
                           c_int32, P, P, c_int32, P], c_int),
        "kvq_decode_workspace": ([POINTER(Cfg), c_int32, c_int32, POINTER(c_size_t)], c_int),
        "kvq_decode_attention": ([POINTER(Cfg), POINTER(CacheStruct), POINTER(CodebookStruct),
                                  POINTER(CodebookStruct), P, P, c_int32, P, P, c_size_t,
                                  c_int32, P], c_int),
        "kvq_dequantize": ([POINTER(Cfg), POINTER(CacheStruct), POINTER(CodebookStruct),
                            POINTER(CodebookStruct), c_int32, c_int32, P, P, P], c_int),
        "kvq_fp16_decode_attention": ([POINTER(Cfg), P, P, c_int32, P, P, P, c_int32, P, P,
                                       c_size_t, c_int32, P], c_int),
        "kvq_fit_workspace": ([c_int32, c_int32, POINTER(c_size_t)], c_int),
        "kvq_fit_codebook": ([P, c_int32, c_int32, c_double, P, c_int32, c_int32, P, P, P,
                              c_size_t, P], c_int),
        "kvq_get_status": ([POINTER(CacheStruct), POINTER(c_int32), P], c_int),
        "kvq_decode_partial": ([POINTER(Cfg), POINTER(CacheStruct), POINTER(CodebookStruct),
                                POINTER(CodebookStruct), P, P, c_int32, c_int32, P, P, P,
                                c_size_t, c_int32, P], c_int),
        "kvq_merge_partials": ([POINTER(Cfg), c_int32, P, P, P, P], c_int),
        "kvq_decode_attention_fused": ([POINTER(Cfg), POINTER(CacheStruct),
                                        POINTER(CodebookStruct), POINTER(CodebookStruct), P, P,
                                        c_int32, P, P, c_size_t, c_int32, P], c_int),
        "kvq_decode_fused_workspace": ([POINTER(Cfg), c_int32, c_int32, POINTER(c_size_t)],
                                       c_int),
        "kvq_quantize_append_noalloc": ([POINTER(Cfg), POINTER(CacheStruct),
                                         POINTER(CodebookStruct), POINTER(CodebookStruct), P, P,
                                         c_int32, P, P], c_int),
        "kvq_step_input_bytes": ([POINTER(Cfg), c_int32, c_int32, POINTER(c_size_t)], c_int),
        "kvq_step_workspace": ([POINTER(Cfg), c_int32, c_int32, c_int32, c_int32,
                                POINTER(c_size_t)], c_int),
        "kvq_step_create": ([POINTER(Cfg), POINTER(StepDesc), POINTER(c_void_p)], c_int),
        "kvq_step_launch": ([P, P, P], c_int),
        "kvq_step_destroy": ([P], c_int),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _check(code: int, where: str) -> None:
    if code != KVQ_OK:
        raise KvqError(code, where)


def _ptr(t):
    return None if t is None else c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return c_void_p(s.cuda_stream)


def make_cfg(B, Hq, Hkv, bits, T_max, outlier_frac, rope_theta, out_cap_k, out_cap_v, D=128):
    return Cfg(B, Hq, Hkv, D, bits, T_max, out_cap_k, out_cap_v, float(outlier_frac),
               float(rope_theta))


def kvq_abi_version() -> int:
    return load().kvq_abi_version()


def kvq_validate_cfg(cfg: Cfg) -> int:
    return load().kvq_validate_cfg(ctypes.byref(cfg))


def kvq_layout(cfg: Cfg) -> dict:
    s = Sizes()
    _check(load().kvq_layout(ctypes.byref(cfg), ctypes.byref(s)), "kvq_layout")
    return {f: getattr(s, f) for f in _CACHE_FIELDS}


class Cache:
    """Device arrays of one layer's cache, allocated with torch per kvq_layout."""

    def __init__(self, cfg: Cfg, device="cuda"):
        import torch
        self.cfg = cfg
        sz = kvq_layout(cfg)
        n = cfg.Hkv * cfg.D
        BW = 16 * cfg.bits                      # words of a 4-token code block
        nq = (cfg.T_max + 3) // 4
        nch = (cfg.T_max + CHUNK - 1) // CHUNK + 1
        dev = torch.device(device)
        i32, f32, f16 = torch.int32, torch.float32, torch.float16
        self.kcodes = torch.zeros((cfg.B, cfg.Hkv, nq, BW), dtype=i32, device=dev)
        self.vcodes = torch.zeros((cfg.B, cfg.Hkv, nq, BW), dtype=i32, device=dev)
        self.kthr = torch.zeros((cfg.B, n, 2), dtype=f16, device=dev)
        self.kparams = torch.zeros((cfg.B, n, 2), dtype=f32, device=dev)
        self.vparams = torch.zeros((cfg.B, cfg.T_max, 2), dtype=f32, device=dev)
        H = cfg.Hkv  # one outlier list per (sequence, kv head)
        self.kout = torch.zeros((cfg.B, H, max(cfg.out_cap_k, 8)), dtype=i32, device=dev)
        self.vout = torch.zeros((cfg.B, H, max(cfg.out_cap_v, 8)), dtype=i32, device=dev)
        self.kchunk = torch.zeros((cfg.B, H, nch), dtype=i32, device=dev)
        self.vchunk = torch.zeros((cfg.B, H, nch), dtype=i32, device=dev)
        self.kcount = torch.zeros((cfg.B, H), dtype=i32, device=dev)
        self.vcount = torch.zeros((cfg.B, H), dtype=i32, device=dev)
        self.len = torch.zeros((cfg.B,), dtype=i32, device=dev)
        self.status = torch.zeros((4,), dtype=i32, device=dev)
        for f in _CACHE_FIELDS:
            assert getattr(self, f).numel() * getattr(self, f).element_size() >= sz[f], f
        self.struct = CacheStruct(*[getattr(self, f).data_ptr() for f in _CACHE_FIELDS])

    def nbytes(self) -> int:
        return sum(getattr(self, f).numel() * getattr(self, f).element_size()
                   for f in _CACHE_FIELDS)


class Codebook:
    """A per-layer NUQ datatype on the device (levels, bounds as float32 tensors)."""

    def __init__(self, levels, bounds):
        self.levels = levels
        self.bounds = bounds
        self.struct = CodebookStruct(levels.data_ptr(), bounds.data_ptr())


def kvq_cache_reset(cache: Cache, stream=None) -> None:
    _check(load().kvq_cache_reset(ctypes.byref(cache.cfg), ctypes.byref(cache.struct),
                                  _stream(stream)), "kvq_cache_reset")


def kvq_quantize_workspace(cfg: Cfg, n_new: int, calibrate: int) -> int:
    b = c_size_t()
    _check(load().kvq_quantize_workspace(ctypes.byref(cfg), n_new, calibrate, ctypes.byref(b)),
           "kvq_quantize_workspace")
    return b.value


def kvq_quantize_append(cache: Cache, cbK: Codebook, cbV: Codebook, k, v, n_new: int, plen,
                        calibrate: int, workspace, stream=None) -> None:
    _check(load().kvq_quantize_append(
        ctypes.byref(cache.cfg), ctypes.byref(cache.struct), ctypes.byref(cbK.struct),
        ctypes.byref(cbV.struct), _ptr(k), _ptr(v), n_new, _ptr(plen), calibrate,
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)),
        "kvq_quantize_append")


def kvq_decode_splits(cfg: Cfg, max_len: int) -> int:
    return load().kvq_decode_splits(ctypes.byref(cfg), max_len)


def kvq_decode_qk_workspace(cfg: Cfg, max_len: int) -> int:
    n = c_size_t()
    _check(load().kvq_decode_qk_workspace(ctypes.byref(cfg), max_len, ctypes.byref(n)),
           "kvq_decode_qk_workspace")
    return n.value


def kvq_decode_qk(cache: Cache, cbK: Codebook, q, qpos, max_len: int, logits, stats, splits: int,
                  workspace, stream=None) -> None:
    _check(load().kvq_decode_qk(ctypes.byref(cache.cfg), ctypes.byref(cache.struct),
                                ctypes.byref(cbK.struct), _ptr(q), _ptr(qpos), max_len,
                                _ptr(logits), _ptr(stats), splits, _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream(stream)),
           "kvq_decode_qk")


def kvq_softmax_merge(cfg: Cfg, stats, splits: int, ml, stream=None) -> None:
    _check(load().kvq_softmax_merge(ctypes.byref(cfg), _ptr(stats), splits, _ptr(ml),
                                    _stream(stream)), "kvq_softmax_merge")


def kvq_decode_pv(cache: Cache, cbV: Codebook, logits, ml, max_len: int, out, part, splits: int,
                  stream=None) -> None:
    _check(load().kvq_decode_pv(ctypes.byref(cache.cfg), ctypes.byref(cache.struct),
                                ctypes.byref(cbV.struct), _ptr(logits), _ptr(ml), max_len,
                                _ptr(out), _ptr(part), splits, _stream(stream)), "kvq_decode_pv")


def kvq_decode_workspace(cfg: Cfg, max_len: int, splits: int) -> int:
    b = c_size_t()
    _check(load().kvq_decode_workspace(ctypes.byref(cfg), max_len, splits, ctypes.byref(b)),
           "kvq_decode_workspace")
    return b.value


def kvq_decode_attention(cache: Cache, cbK: Codebook, cbV: Codebook, q, qpos, max_len: int, out,
                         workspace, splits: int = 0, stream=None) -> None:
    _check(load().kvq_decode_attention(
        ctypes.byref(cache.cfg), ctypes.byref(cache.struct), ctypes.byref(cbK.struct),
        ctypes.byref(cbV.struct), _ptr(q), _ptr(qpos), max_len, _ptr(out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), splits, _stream(stream)),
        "kvq_decode_attention")


def kvq_decode_fused_workspace(cfg: Cfg, max_len: int, splits: int) -> int:
    b = c_size_t()
    _check(load().kvq_decode_fused_workspace(ctypes.byref(cfg), max_len, splits, ctypes.byref(b)),
           "kvq_decode_fused_workspace")
    return b.value


def kvq_decode_attention_fused(cache: Cache, cbK: Codebook, cbV: Codebook, q, qpos, max_len: int,
                               out, workspace, splits: int = 0, stream=None) -> None:
    _check(load().kvq_decode_attention_fused(
        ctypes.byref(cache.cfg), ctypes.byref(cache.struct), ctypes.byref(cbK.struct),
        ctypes.byref(cbV.struct), _ptr(q), _ptr(qpos), max_len, _ptr(out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), splits, _stream(stream)),
        "kvq_decode_attention_fused")


def kvq_decode_partial(cache: Cache, cbK: Codebook, cbV: Codebook, q, qpos, max_len: int,
                       pos_offset: int, ml, o, workspace, splits: int = 0, stream=None) -> None:
    _check(load().kvq_decode_partial(
        ctypes.byref(cache.cfg), ctypes.byref(cache.struct), ctypes.byref(cbK.struct),
        ctypes.byref(cbV.struct), _ptr(q), _ptr(qpos), max_len, pos_offset, _ptr(ml), _ptr(o),
        _ptr(workspace), workspace.numel() * workspace.element_size(), splits, _stream(stream)),
        "kvq_decode_partial")


def kvq_merge_partials(cfg: Cfg, parts: int, ml, o, out, stream=None) -> None:
    _check(load().kvq_merge_partials(ctypes.byref(cfg), parts, _ptr(ml), _ptr(o), _ptr(out),
                                     _stream(stream)), "kvq_merge_partials")


def kvq_dequantize(cache: Cache, cbK: Codebook, cbV: Codebook, t0: int, nt: int, khat, vhat,
                   stream=None) -> None:
    _check(load().kvq_dequantize(ctypes.byref(cache.cfg), ctypes.byref(cache.struct),
                                 ctypes.byref(cbK.struct), ctypes.byref(cbV.struct), t0, nt,
                                 _ptr(khat), _ptr(vhat), _stream(stream)), "kvq_dequantize")


def kvq_fp16_decode_attention(cfg: Cfg, K, V, T_stride: int, lens, q, qpos, max_len: int, out,
                              workspace, splits: int = 0, stream=None) -> None:
    _check(load().kvq_fp16_decode_attention(
        ctypes.byref(cfg), _ptr(K), _ptr(V), T_stride, _ptr(lens), _ptr(q), _ptr(qpos), max_len,
        _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(), splits,
        _stream(stream)), "kvq_fp16_decode_attention")


def kvq_fit_workspace(n_vec: int, vec_len: int) -> int:
    b = c_size_t()
    _check(load().kvq_fit_workspace(n_vec, vec_len, ctypes.byref(b)), "kvq_fit_workspace")
    return b.value


def kvq_fit_codebook(samples, f: float, bits: int, levels, bounds, workspace, weights=None,
                     max_iter: int = 100, stream=None) -> None:
    n_vec, vec_len = samples.shape
    _check(load().kvq_fit_codebook(_ptr(samples), n_vec, vec_len, float(f), _ptr(weights), bits,
                                   max_iter, _ptr(levels), _ptr(bounds), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)),
           "kvq_fit_codebook")


def kvq_quantize_append_noalloc(cache: Cache, cbK: Codebook, cbV: Codebook, k, v, n_new: int,
                                plen=None, stream=None) -> None:
    """Append without a workspace: the library's own fixed device scratch is used instead."""
    _check(load().kvq_quantize_append_noalloc(
        ctypes.byref(cache.cfg), ctypes.byref(cache.struct), ctypes.byref(cbK.struct),
        ctypes.byref(cbV.struct), _ptr(k), _ptr(v), n_new, _ptr(plen), _stream(stream)),
        "kvq_quantize_append_noalloc")


def kvq_step_input_bytes(cfg: Cfg, layers: int, n_new: int) -> int:
    b = c_size_t()
    _check(load().kvq_step_input_bytes(ctypes.byref(cfg), layers, n_new, ctypes.byref(b)),
           "kvq_step_input_bytes")
    return b.value


def kvq_step_workspace(cfg: Cfg, n_new: int, max_len: int, splits: int = 0,
                       fused: int = 0) -> int:
    b = c_size_t()
    _check(load().kvq_step_workspace(ctypes.byref(cfg), n_new, max_len, splits, fused,
                                     ctypes.byref(b)), "kvq_step_workspace")
    return b.value


class Step:
    """Handle of a recorded whole-model step (kvq_step_create); keeps its buffers alive."""

    def __init__(self, handle, keep):
        self.handle = handle
        self._keep = keep

    def destroy(self) -> None:
        if self.handle:
            _check(load().kvq_step_destroy(self.handle), "kvq_step_destroy")
            self.handle = None


def kvq_step_create(cfg: Cfg, caches, cbK, cbV, n_new: int, max_len: int, inputs, out,
                    workspace, splits: int = 0, fused: int = 0) -> Step:
    """caches, cbK, cbV: one Cache / Codebook per layer, in layer order."""
    L = len(caches)
    if len(cbK) != L or len(cbV) != L:
        raise ValueError(f"kvq_step_create: {L} caches but {len(cbK)} key and {len(cbV)} value "
                         "codebooks")
    carr = (CacheStruct * L)(*[c.struct for c in caches])
    karr = (CodebookStruct * L)(*[c.struct for c in cbK])
    varr = (CodebookStruct * L)(*[c.struct for c in cbV])
    desc = StepDesc(L, carr, karr, varr, n_new, max_len, splits, fused, inputs.data_ptr(),
                    out.data_ptr(), workspace.data_ptr(),
                    workspace.numel() * workspace.element_size())
    h = c_void_p()
    _check(load().kvq_step_create(ctypes.byref(cfg), ctypes.byref(desc), ctypes.byref(h)),
           "kvq_step_create")
    return Step(h, (inputs, out, workspace, list(caches), list(cbK), list(cbV)))


def kvq_step_launch(step: Step, inputs=None, stream=None) -> None:
    """inputs: a packed input record (host or device tensor), or None if already in place."""
    _check(load().kvq_step_launch(step.handle, _ptr(inputs), _stream(stream)),
           "kvq_step_launch")


def kvq_step_destroy(step: Step) -> None:
    step.destroy()


def kvq_get_status(cache: Cache, stream=None) -> int:
    out = c_int32()
    _check(load().kvq_get_status(ctypes.byref(cache.struct), ctypes.byref(out), _stream(stream)),
           "kvq_get_status")
    return out.value
