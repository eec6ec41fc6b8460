"""Shared builders for the GPU parity tests (not collected as tests)."""
from __future__ import annotations

import numpy as np

import oracle as O
import synth


def host_block(w, T, layer=0):
    """fp16 K, V [B, T, Hkv, D] from the numpy generator."""
    idx = (np.arange(w.B)[:, None, None, None], np.arange(T)[None, :, None, None],
           np.arange(w.Hkv)[None, None, :, None], np.arange(w.D)[None, None, None, :])
    return synth.gen_k(w, layer, *idx), synth.gen_v(w, layer, *idx)


def oracle_codebooks(w, layer=0):
    cbK = O.fit_codebook(synth.codebook_samples_k(w, layer), w.f, w.bits)
    cbV = O.fit_codebook(synth.codebook_samples_v(w, layer), w.f, w.bits)
    return cbK, cbV


def to_dev_codebook(cb):
    import torch
    import long_context_decode_nuq_b200 as K
    lev = torch.from_numpy(np.ascontiguousarray(cb[0], dtype=np.float32)).cuda()
    bnd = torch.from_numpy(np.ascontiguousarray(cb[1], dtype=np.float32)).cuda()
    return K.Codebook(lev, bnd)


def gpu_cache(w, T_max, cap_k, cap_v):
    import long_context_decode_nuq_b200 as K
    cfg = K.make_cfg(w.B, w.Hq, w.Hkv, w.bits, T_max, w.f, w.rope_theta, cap_k, cap_v)
    c = K.Cache(cfg)
    K.kvq_cache_reset(c)
    return c


def gpu_quantize(cache, cbK, cbV, K16, V16, plen=None, calibrate=0):
    """K16, V16: numpy fp16 [B, n, Hkv, D] (or torch cuda fp16)."""
    import torch
    import long_context_decode_nuq_b200 as K
    k = torch.as_tensor(K16).cuda() if not torch.is_tensor(K16) else K16
    v = torch.as_tensor(V16).cuda() if not torch.is_tensor(V16) else V16
    n_new = k.shape[1]
    pl = None if plen is None else torch.tensor(np.asarray(plen, dtype=np.int32)).cuda()
    ws = torch.empty(K.kvq_quantize_workspace(cache.cfg, n_new, calibrate), dtype=torch.uint8,
                     device="cuda")
    K.kvq_quantize_append(cache, cbK, cbV, k.contiguous(), v.contiguous(), n_new, pl, calibrate,
                          ws)
    torch.cuda.synchronize()


def u32(t):
    return t.cpu().numpy().view(np.uint32)


def u16(t):
    return t.cpu().numpy().view(np.uint16)


def same_f32(a, b):
    """Bit-for-bit equality of binary32 arrays, except that a NaN matches any NaN: IEEE 754
    leaves the payload of an operation's NaN result open, so only NaN-ness is compared."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    b = np.ascontiguousarray(b, dtype=np.float32)
    if a.shape != b.shape:
        return False
    return bool(np.all((np.isnan(a) & np.isnan(b)) | (a.view(np.uint32) == b.view(np.uint32))))


def compare_cache(g, o, B, hard=True):
    """Bit-exact comparison of a GPU cache with the oracle's QuantizedCache."""
    errs = []
    glen = g.len.cpu().numpy()
    if not np.array_equal(glen, o.len):
        errs.append(f"len {glen} vs {o.len}")
    for b in range(B):
        L = int(o.len[b])
        for name, n_rows in (("kcodes", (L + 3) // 4), ("vcodes", (L + 3) // 4)):
            gv = u32(getattr(g, name)[b, :, :n_rows])
            ov = getattr(o, name)[b, :, :n_rows]
            if not np.array_equal(gv, ov):
                bad = np.argwhere(gv != ov)
                errs.append(f"{name}[b={b}] {len(bad)} words differ, first {bad[:3].tolist()}")
        if L > 0 or True:
            if not np.array_equal(u16(g.kthr[b]), o.kthr[b]):
                errs.append(f"kthr[b={b}]")
            if not same_f32(g.kparams[b].cpu().numpy(), o.kparams[b]):
                errs.append(f"kparams[b={b}]")
        if not same_f32(g.vparams[b, :L].cpu().numpy(), o.vparams[b, :L]):
            errs.append(f"vparams[b={b}]")
        for s in ("k", "v"):
            nch = (L + 63) // 64
            for h in range(o.Hkv):
                cnt = int(o.out_count[s][b, h])
                gcnt = int(u32(getattr(g, f"{s}count"))[b, h])
                if gcnt != cnt:
                    errs.append(f"{s}count[b={b},h={h}] {gcnt} vs {cnt}")
                    continue
                if not np.array_equal(u32(getattr(g, f"{s}out")[b, h, :cnt]), o.out[s][b, h, :cnt]):
                    errs.append(f"{s}out[b={b},h={h}]")
                gch = u32(getattr(g, f"{s}chunk")[b, h, : nch + 1])
                if not np.array_equal(gch, o.chunk_ptr[s][b, h, : nch + 1]):
                    errs.append(f"{s}chunk[b={b},h={h}] {gch[:8]} vs {o.chunk_ptr[s][b, h, :nch+1][:8]}")
    st = int(g.status.cpu().numpy()[0])
    if st != o.status:
        errs.append(f"status {st} vs {o.status}")
    if hard:
        assert not errs, "\n".join(errs)
    return errs
