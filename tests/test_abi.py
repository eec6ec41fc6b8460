"""The C-ABI library loads, exports every declared symbol and rejects bad arguments
before touching the GPU (no compute calls here)."""
import ctypes
import os
import re

import pytest

import long_context_decode_nuq_b200 as K

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "kvq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = K.load()
    names = _declared()
    assert len(names) >= 18
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(K.EXPORTS)
    assert K.kvq_abi_version() == 2


def test_cfg_validation():
    ok = K.make_cfg(1, 32, 32, 3, 4096, 0.01, 1e4, 104, 104)
    assert K.kvq_validate_cfg(ok) == 0
    bad = [
        dict(bits=5), dict(bits=1), dict(D=64), dict(Hq=30), dict(B=0), dict(T_max=0),
        dict(outlier_frac=1.5), dict(rope_theta=0.5), dict(out_cap_k=-1), dict(out_cap_v=12),
    ]
    for kw in bad:
        args = dict(B=1, Hq=32, Hkv=32, bits=3, T_max=4096, outlier_frac=0.01, rope_theta=1e4,
                    out_cap_k=104, out_cap_v=104, D=128)
        args.update(kw)
        assert K.kvq_validate_cfg(K.make_cfg(**args)) < 0, kw
    assert K.load().kvq_validate_cfg(None) == -1


def test_layout_sizes():
    cfg = K.make_cfg(2, 8, 4, 3, 1000, 0.01, 1e4, 48, 72)
    s = K.kvq_layout(cfg)
    assert s["kcodes"] == 2 * 1000 * 4 * 12 * 4 and s["vcodes"] == s["kcodes"]
    # code blocks hold four tokens: T_max is rounded up to a multiple of 4
    s2 = K.kvq_layout(K.make_cfg(2, 8, 4, 3, 1001, 0.01, 1e4, 48, 72))
    assert s2["kcodes"] == s2["vcodes"] == 2 * 251 * 4 * 48 * 4
    assert s["vparams"] == 2 * 1000 * 2 * 4
    # one outlier list per (sequence, kv head)
    assert s["kout"] == 2 * 4 * 48 * 4 and s["vout"] == 2 * 4 * 72 * 4
    assert s["kchunk"] == 2 * 4 * (16 + 1) * 4 and s["kcount"] == 2 * 4 * 4
    assert K.kvq_quantize_workspace(cfg, 100, 1) > K.kvq_quantize_workspace(cfg, 100, 0)
    assert K.kvq_decode_splits(cfg, 1000) >= 1


def test_argument_errors_without_gpu():
    lib = K.load()
    cfg = K.make_cfg(1, 4, 4, 3, 256, 0.01, 1e4, 64, 64)
    empty = K.CacheStruct()
    cb = K.CodebookStruct(None, None)
    null = None
    # NULL cache arrays are rejected synchronously
    rc = lib.kvq_quantize_append(ctypes.byref(cfg), ctypes.byref(empty), ctypes.byref(cb),
                                 ctypes.byref(cb), null, null, 1, null, 0, null, 0, null)
    assert rc == -1
    # misaligned (never dereferenced) pointers are rejected
    fake = K.CacheStruct(*([0x1000] * 13))
    fake.kcodes = 0x1001
    rc = lib.kvq_cache_reset(ctypes.byref(cfg), ctypes.byref(fake), null)
    assert rc == -2
    # unsupported head_dim is reported before anything else
    cfg64 = K.make_cfg(1, 4, 4, 3, 256, 0.01, 1e4, 64, 64, D=64)
    assert lib.kvq_cache_reset(ctypes.byref(cfg64), ctypes.byref(fake), null) == -4
    # split count out of range
    fake.kcodes = 0x1000
    cbf = K.CodebookStruct(0x1000, 0x1000)
    rc = lib.kvq_decode_qk(ctypes.byref(cfg), ctypes.byref(fake), ctypes.byref(cbf), 0x1000,
                           0x1000, 100, 0x1000, 0x1000, 5000, 0x1000, 1 << 20, null)
    assert rc == -5
    # fit: too many samples
    assert lib.kvq_fit_workspace(5, 5000, ctypes.byref(ctypes.c_size_t())) == -3
    assert K.load().kvq_strerror(-6) == b"workspace too small"


def test_noalloc_append_argument_errors_without_gpu():
    lib = K.load()
    null = None
    cfg = K.make_cfg(1, 4, 4, 3, 256, 0.01, 1e4, 64, 64)
    cb = K.CodebookStruct(0x1000, 0x1000)
    empty = K.CacheStruct()
    rc = lib.kvq_quantize_append_noalloc(ctypes.byref(cfg), ctypes.byref(empty), ctypes.byref(cb),
                                         ctypes.byref(cb), 0x1000, 0x1000, 1, null, null)
    assert rc == -1
    # a request whose scratch exceeds the fixed array is refused before any device work
    big = K.make_cfg(64, 32, 32, 3, 8192, 0.01, 1e4, 64, 64)
    assert K.kvq_quantize_workspace(big, 4096, 0) > K.NOALLOC_SCRATCH_BYTES
    fake = K.CacheStruct(*([0x1000] * 13))
    rc = lib.kvq_quantize_append_noalloc(ctypes.byref(big), ctypes.byref(fake), ctypes.byref(cb),
                                         ctypes.byref(cb), 0x1000, 0x1000, 4096, null, null)
    assert rc == -8
    assert b"scratch" in lib.kvq_strerror(-8)
    # n_new beyond T_max is a range error, checked before the scratch size
    rc = lib.kvq_quantize_append_noalloc(ctypes.byref(cfg), ctypes.byref(fake), ctypes.byref(cb),
                                         ctypes.byref(cb), 0x1000, 0x1000, 257, null, null)
    assert rc == -5


def test_step_sizes_and_argument_errors_without_gpu():
    """The whole-model step's record size is the closed form of its packed layout, and bad
    descriptors are refused before any CUDA call."""
    lib = K.load()
    cfg = K.make_cfg(2, 8, 4, 3, 512, 0.01, 1e4, 64, 64)
    # per layer: k and v fp16 [B][n_new][Hkv][D], q fp16 [B][Hq][D]; then qpos int32 [B]
    # padded to 16 bytes
    assert K.kvq_step_input_bytes(cfg, 3, 1) == 3 * (2 * 2 * 1 * 4 * 128 * 2 + 2 * 8 * 128 * 2) + 16
    assert K.kvq_step_input_bytes(cfg, 1, 0) == 2 * 8 * 128 * 2 + 16
    assert K.kvq_step_input_bytes(cfg, 2, 5) == 2 * (2 * 2 * 5 * 4 * 128 * 2 + 2 * 8 * 128 * 2) + 16
    ws = K.kvq_step_workspace(cfg, 1, 400)
    assert ws >= K.kvq_decode_workspace(cfg, 400, 0)
    assert ws >= K.kvq_quantize_workspace(cfg, 1, 0)
    assert K.kvq_step_workspace(cfg, 0, 400) == K.kvq_decode_workspace(cfg, 400, 0)
    n = ctypes.c_size_t()
    assert lib.kvq_step_input_bytes(ctypes.byref(cfg), 0, 1, ctypes.byref(n)) == -3
    assert lib.kvq_step_input_bytes(ctypes.byref(cfg), 1, -1, ctypes.byref(n)) == -3
    assert lib.kvq_step_workspace(ctypes.byref(cfg), 1, 400, 0, 2, ctypes.byref(n)) == -3
    # fused attention needs one query head per kv head
    assert lib.kvq_step_workspace(ctypes.byref(cfg), 1, 400, 0, 1, ctypes.byref(n)) == -4

    caches = (K.CacheStruct * 1)()
    cbs = (K.CodebookStruct * 1)()
    h = ctypes.c_void_p()

    def desc(**kw):
        d = dict(layers=1, caches=caches, cbK=cbs, cbV=cbs, n_new=1, max_len=400, splits=0,
                 fused=0, inputs=0x10000, out=0x20000, workspace=0x30000, workspace_bytes=ws)
        d.update(kw)
        return K.StepDesc(**d)

    def create(d):
        return lib.kvq_step_create(ctypes.byref(cfg), ctypes.byref(d), ctypes.byref(h))

    assert lib.kvq_step_create(ctypes.byref(cfg), None, ctypes.byref(h)) == -1
    assert create(desc(inputs=None)) == -1 and h.value is None
    assert create(desc(out=0x20004)) == -2
    assert create(desc(workspace=0x30008)) == -2
    assert create(desc(layers=0)) == -3
    assert create(desc(max_len=600)) < 0      # past T_max
    assert create(desc(workspace_bytes=ws - 16)) == -6
    assert lib.kvq_step_launch(None, None, None) == -1
    assert lib.kvq_step_destroy(None) == -1


def test_step_binding_checks_layer_lists():
    """The binding refuses per-layer lists of different lengths before calling the library."""
    cfg = K.make_cfg(1, 4, 4, 3, 256, 0.01, 1e4, 64, 64)

    class _Fake:
        struct = K.CacheStruct()

    with pytest.raises(ValueError):
        K.kvq_step_create(cfg, [_Fake(), _Fake()], [_Fake()], [_Fake(), _Fake()], 1, 200,
                          None, None, None)
