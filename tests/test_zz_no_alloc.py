"""The allocation-free append entry point against the workspace one.

Collected last on purpose: the no-alloc entry point keeps one scratch array per device
for the life of the process, so this file also shows that it works after every other
GPU test has run in the same process (and it passes when run alone).
"""
import numpy as np
import pytest

import synth
from kvq_testlib import gpu_cache, gpu_quantize, host_block, oracle_codebooks, to_dev_codebook, u16, u32

pytestmark = pytest.mark.gpu


def _arrays(c, B):
    out = {}
    for name in ("kcodes", "vcodes", "kparams", "vparams", "kout", "vout", "kchunk",
                 "vchunk", "kcount", "vcount", "len", "status"):
        t = getattr(c, name)
        out[name] = t.cpu().numpy().copy()
    for name in ("kthr",):
        out[name] = u16(getattr(c, name)).copy()
    return out


def _same(a, b):
    bad = [k for k in a if not np.array_equal(a[k].view(np.uint8), b[k].view(np.uint8))]
    assert not bad, f"arrays differ: {bad}"


@pytest.mark.parametrize("name,bits", [("llama3_8b_gqa_128k", 3), ("batched_8x8k", 2)])
def test_noalloc_append_matches_workspace_append(name, bits):
    import torch
    import long_context_decode_nuq_b200 as K

    w = synth.workload(name, B=3, T=300, bits=bits)
    T_max = 512
    # two appends of n = 37 and 64 tokens; the second one ragged over the batch
    appends = [(37, None), (64, [64, 13, 0])]
    total = w.T + sum(n for n, _ in appends)
    K16, V16 = host_block(w, total)
    cbK, cbV = (to_dev_codebook(cb) for cb in oracle_codebooks(w))
    cap = 1 << 16  # room for every outlier: the status word must stay 0
    ref = gpu_cache(w, T_max, cap, cap)
    new = gpu_cache(w, T_max, cap, cap)
    for c in (ref, new):
        gpu_quantize(c, cbK, cbV, K16[:, : w.T], V16[:, : w.T], calibrate=1)
    _same(_arrays(ref, w.B), _arrays(new, w.B))
    t = w.T
    for n, plen in appends:
        k = torch.as_tensor(K16[:, t : t + n]).cuda().contiguous()
        v = torch.as_tensor(V16[:, t : t + n]).cuda().contiguous()
        pl = None if plen is None else torch.tensor(np.asarray(plen, np.int32)).cuda()
        gpu_quantize(ref, cbK, cbV, k, v, plen=plen)
        K.kvq_quantize_append_noalloc(new, cbK, cbV, k, v, n, pl)
        torch.cuda.synchronize()
        _same(_arrays(ref, w.B), _arrays(new, w.B))
        t += n
    assert K.kvq_get_status(new) == 0
    assert list(new.len.cpu().numpy()) == [w.T + 37 + 64, w.T + 37 + 13, w.T + 37]


def test_noalloc_append_refuses_oversize_request():
    import torch
    import long_context_decode_nuq_b200 as K

    w = synth.workload("tiny_single_head", B=8)
    cache = gpu_cache(w, 8192, 16, 16)
    assert K.kvq_quantize_workspace(cache.cfg, 8192, 0) > K.NOALLOC_SCRATCH_BYTES
    k = torch.zeros(8, 8192, 1, 128, dtype=torch.float16, device="cuda")
    cb = K.Codebook(torch.zeros(8, device="cuda"), torch.zeros(7, device="cuda"))
    with pytest.raises(K.KvqError):
        K.kvq_quantize_append_noalloc(cache, cb, cb, k, k, 8192)
    torch.cuda.synchronize()
    assert int(cache.len.cpu().sum()) == 0
