"""Pins of bench.py's byte model (every GB/s and roofline fraction the bench reports rests on it).

What fixes the expected values:
  * tests/golden/compression_ratio.txt -- the pages' cache reduction of a 3-bit cache against
    fp16 (phantomic12 research note, "Paper's own claim": about 5.3x), which is 16/3 when the
    scales and outliers are left out;
  * tests/golden/context_capacity.txt -- the pages' capacity claim (study.space summary and the
    phantomic12 note: LLaMA-7B at up to 1M tokens of context on one A100-80GB);
  * the per-token closed form of the decode's algorithmic bytes, written out below term by
    term: K and V codes n*b/8 each, one entry per outlier (f*n key entries, 2*k_v value entries,
    k_v = floor(f*n/2 + 1/2)), 8 B of value (off, half) per token, and -- for the split path
    only -- 4 B per query head each way for the fp32 logits.  With the 6-byte outlier entry of a
    (position, fp16 value) pair this gives the per-configuration figures 124 / 3566 / 2542 /
    3566 / 4590 / 897 / 3323 B per token per layer; this library's entries are one packed
    uint32 (4 B), which the model counts by default.
"""
import math
import os

import pytest

import bench
import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _read(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split()
            out[k] = float(v)
    return out


def test_ratio_16_over_3_at_zero_overheads():
    g = _read("compression_ratio.txt")
    w = synth.workload("llama7b_layer_32k", bits=int(g["bits_code"]), f=0.0)
    fp16_bytes = 2 * w.n * g["bits_fp16"] / 8           # K and V rows in fp16
    q_bytes = bench.cache_bytes_per_token(w, params=False)
    assert fp16_bytes / q_bytes == pytest.approx(g["ratio_num"] / g["ratio_den"], rel=0, abs=1e-12)
    assert round(fp16_bytes / q_bytes, 1) == g["ratio_rounded_1dp"]
    # the outliers and value scales only lower the ratio
    w1 = synth.workload("llama7b_layer_32k", bits=3, f=0.01)
    assert fp16_bytes / bench.cache_bytes_per_token(w1) < fp16_bytes / q_bytes


@pytest.mark.parametrize("name,over,expect", [
    ("tiny_single_head", {}, 124),
    ("llama7b_layer_32k", {}, 3566),
    ("batched_8x8k", dict(bits=2), 2542),
    ("batched_8x8k", dict(bits=3), 3566),
    ("batched_8x8k", dict(bits=4), 4590),
    ("llama3_8b_gqa_128k", {}, 897),
    ("llama7b_1m_32layers", {}, 3323),
])
def test_closed_form_per_token(name, over, expect):
    w = synth.workload(name, **over)
    got = bench.cache_bytes_per_token(w, outlier_bytes=6)
    assert round(got) == expect
    # the decode traffic per token equals the stored bytes plus the chunk pointers (one uint32
    # per 64 tokens per kv head, K and V) for the fused path, and adds the logits (4 B per
    # query head, written then read) for the split kernels (three calls or one)
    # (outlier counts are totals over the batch's w.B sequences)
    T = 1 << 16
    BT = w.B * T
    k_out, v_out = bench.expected_outliers_per_token(w)
    fused = bench.bytes_model(w, T, k_out * BT, v_out * BT, "fused", outlier_bytes=6)["total"]
    ptr = 2 * 4 * w.Hkv * ((T + 63) // 64 + 1) * w.B
    assert (fused - ptr) / BT == pytest.approx(got, rel=1e-12)
    split = bench.bytes_model(w, T, k_out * BT, v_out * BT, "split", outlier_bytes=6)
    assert split["total"] - fused == 2 * 4 * w.Hq * BT
    assert split["qk"] + split["pv"] == split["total"]
    one = bench.bytes_model(w, T, k_out * BT, v_out * BT, "one-call", outlier_bytes=6)["total"]
    assert one == split["total"]


def test_default_counts_one_packed_word_per_outlier():
    w = synth.workload("llama7b_1m_32layers")
    k_out, v_out = bench.expected_outliers_per_token(w)
    assert k_out == pytest.approx(0.005 * 4096) and v_out == 2 * math.floor(0.005 * 4096 / 2 + 0.5)
    assert bench.cache_bytes_per_token(w) == pytest.approx(3072 + 4 * (k_out + v_out) + 8)
    # the whole 32-layer cache at 2^20 tokens: about 111.5 GB with 6-byte entries
    total6 = bench.cache_bytes_per_token(w, outlier_bytes=6) * w.layers * w.T
    assert total6 / 1e9 == pytest.approx(111.5, abs=0.1)


def test_capacity_claim_bounds_the_bit_width():
    g = _read("context_capacity.txt")
    shape = dict(Hq=int(g["kv_heads"]), Hkv=int(g["kv_heads"]), D=int(g["head_dim"]), f=0.0)
    per_gpu = g["gpu_bytes"]
    tokens, layers = g["tokens"], g["layers"]
    fits = {}
    for bits in (2, 3, 4):
        w = synth.workload("llama7b_layer_32k", bits=bits, **shape)
        fits[bits] = bench.cache_bytes_per_token(w, params=False) * layers * tokens <= per_gpu
    # codes alone: 2 bits fit 80 GB at 1M tokens (65.5 GB), 3 and 4 bits do not (98.3, 131 GB);
    # the claim therefore needs about 2-bit codes, and an fp16 cache (524 GB) is far outside
    assert fits == {2: True, 3: False, 4: False}
    w16 = synth.workload("llama7b_layer_32k", **shape)
    assert 2 * w16.n * 2 * layers * tokens > 6 * per_gpu
