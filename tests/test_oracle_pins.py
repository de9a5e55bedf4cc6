"""The sizes the pages print, checked against the oracle's formats (CPU only).

Values and their sources live in tests/golden/page_sizes.txt.
"""
import os

from oracle import layout, quant
from synth import WORKLOADS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_sizes.txt")


def _golden():
    out = {}
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = line.split()
            out[k] = int(v)
    return out


def test_sizes_printed_on_the_pages():
    g = _golden()
    w = WORKLOADS["decode131k"]
    per_token = w.layers * w.kv_heads * 256
    assert per_token == g["elements_per_token"]
    assert 65536 * per_token * 2 * 2 == g["f16_kv_bytes_per_65536_tokens"]
    bpe_q4 = quant.block_bytes("q4_0") / 32
    assert per_token * 2 * bpe_q4 == g["q4_0_kv_bytes_per_token"]
    assert quant.block_bytes("q8_0") * 8 * 2 // 32 == g["q8_0_bits_per_element_x2"]
    assert quant.block_bytes("q5_1") * 8 / 32 == g["q5_1_bits_per_element"]
    assert round(100 * (quant.block_bytes("q5_1") / quant.block_bytes("q4_0") - 1)) == g["q5_1_over_q4_0_key_bits_pct"]
    bt = g["block_tokens"]
    assert 62080 // bt == g["blocks_in_62080_tokens"] and 62080 % bt == 0
    assert 32768 // bt == g["blocks_in_budget_32768"]
    assert 8192 // bt == g["blocks_in_budget_8192"]
    assert round(100 * 256 / 485) == g["coverage_pct_budget_32768"]
    assert round(100 * 64 / 485) == g["coverage_pct_budget_8192"]
    assert 16384 // bt == g["blocks_in_reserve_16384"]


def test_page_sizes_follow_block_sizes():
    assert layout.page_bytes("k", "q8_0") == 128 * 8 * quant.block_bytes("q8_0") == 34816
    assert layout.page_bytes("v", "q4_0") == 128 * 8 * quant.block_bytes("q4_0") == 18432
    assert layout.page_bytes("v", "q8_0") == 34816
    assert layout.page_bytes("k", "q4_0") == 18432
    assert layout.page_bytes("k", "q5_1") == 128 * 8 * quant.block_bytes("q5_1") == 24576
    assert layout.page_bytes("k", "q5_0") == 128 * 8 * quant.block_bytes("q5_0") == 22528
    assert layout.page_bytes("v", "q4_1") == 128 * 8 * quant.block_bytes("q4_1") == 20480


def test_decode_bytes_per_step():
    # 131,072 tokens x 16 layers x 4 KV heads x (272 B of K + 144 B of V) per token-head.
    w = WORKLOADS["decode131k"]
    per = (layout.page_bytes("k", "q8_0") + layout.page_bytes("v", "q4_0")) // 128
    assert per == 416
    assert w.context * w.layers * w.kv_heads * per == 3_489_660_928
