"""Device-side fill of the synthetic inputs (binding of libkvqsynth.so, built from gen.cu).

Produces exactly the fp16 values of ``philox.gen_k / gen_v / gen_q`` directly in
GPU memory, for workloads too large to generate on the host.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import c_double, c_int, c_uint32, c_uint64, c_void_p

import numpy as np

from . import philox as P

LIB = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkvqsynth.so")
_lib = None


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise ImportError(f"{LIB} missing; run python -m long_context_decode_nuq_b200.build")
        lib = ctypes.CDLL(LIB)
        lib.kvqsynth_fill_kv.argtypes = [c_uint32, c_uint32, c_uint32, c_int, c_int, c_int, c_int,
                                         c_int, c_int, c_void_p, c_void_p, c_uint32, c_double,
                                         c_void_p, c_void_p]
        lib.kvqsynth_fill_kv.restype = c_int
        lib.kvqsynth_fill_normal.argtypes = [c_uint32, c_uint32, c_uint32, c_uint64, c_uint64,
                                             c_void_p, c_void_p]
        lib.kvqsynth_fill_normal.restype = c_int
        _lib = lib
    return _lib


class DeviceGen:
    """Per (workload, layer) device generator; holds the per-channel tables on the GPU."""

    def __init__(self, w: P.Workload, layer: int = 0, device="cuda"):
        import torch
        self.w, self.layer = w, layer
        self.scale = torch.from_numpy(P.heavy_channel_scale(w, layer).reshape(-1).copy()).to(device)
        tm = P.student_t_channels(w, layer).reshape(-1).astype(np.uint8)
        self.tmask = torch.from_numpy(tm).to(device) if tm.any() else None

    def _stream(self):
        import torch
        return c_void_p(torch.cuda.current_stream().cuda_stream)

    def fill_k(self, out, t0: int, nt: int) -> None:
        w = self.w
        rc = _load().kvqsynth_fill_kv(w.seed, self.layer, P.STREAM_K, w.B, w.T_gen, w.Hkv, w.D,
                                     t0, nt, c_void_p(self.scale.data_ptr()),
                                     c_void_p(self.tmask.data_ptr()) if self.tmask is not None
                                     else None, 0, 1.0, c_void_p(out.data_ptr()), self._stream())
        assert rc == 0, rc

    def fill_v(self, out, t0: int, nt: int) -> None:
        w = self.w
        thr = P.spike_threshold(w.v_spike_p) if w.v_spike_p > 0 else 0
        rc = _load().kvqsynth_fill_kv(w.seed, self.layer, P.STREAM_V, w.B, w.T_gen, w.Hkv, w.D,
                                     t0, nt, None, None, thr, float(w.v_spike_scale),
                                     c_void_p(out.data_ptr()), self._stream())
        assert rc == 0, rc

    def fill_q(self, out, step: int = 0) -> None:
        w = self.w
        n = w.B * w.Hq * w.D
        rc = _load().kvqsynth_fill_normal(w.seed, self.layer, P.STREAM_Q, step * n, n,
                                         c_void_p(out.data_ptr()), self._stream())
        assert rc == 0, rc
