"""Pins for oracle.sizing: the pages' worked sizing numbers."""
from oracle.sizing import kv_bytes, blocks_for, block_bytes, decode_kv_bytes


def test_13b_example():
    # 40 layers, hidden 5120 = 40 heads x 128, fp16: roughly 819 KB per token,
    # about 1.6 GB for a 2,000-token conversation, about 26 GB for 16 of them.
    per_tok = kv_bytes(40, 40, 128, 1, 2)
    assert per_tok == 2 * 40 * 5120 * 2 == 819_200
    assert kv_bytes(40, 40, 128, 2000, 2) == 1_638_400_000
    assert round(kv_bytes(40, 40, 128, 2000, 2, batch=16) / 1e9) == 26
    # capacity planning: ~54 GB at ~819 KB/token is roughly 66,000 tokens,
    # about 33 sequences of 2,000 tokens or ~8 of 8,000
    tokens_max = 54e9 / per_tok
    assert round(tokens_max, -3) == 66_000
    assert round(tokens_max / 2000) == 33 and int(tokens_max / 8000) == 8


def test_llama3_70b_example():
    per_tok = kv_bytes(80, 8, 128, 1, 2)
    assert per_tok == 327_680
    total = kv_bytes(80, 8, 128, 4096, 2, batch=64)
    assert total == 85_899_345_920 == 80 * 2 ** 30       # the page prints 83.88 "GB"
    assert kv_bytes(1, 8, 128, 4096, 2, batch=64) == 1_073_741_824   # one layer


def test_levers_and_blocks():
    assert kv_bytes(32, 32, 128, 100, 2) == 4 * kv_bytes(32, 8, 128, 100, 2)   # 4x GQA ratio
    assert kv_bytes(32, 8, 128, 100, 1) * 2 == kv_bytes(32, 8, 128, 100, 2)    # fp8 halves
    assert blocks_for(25, 16) == 2 and blocks_for(32, 16) == 2 and blocks_for(33, 16) == 3
    assert block_bytes(16, 8, 128, 2) == 65_536                                 # K+V, one layer
    assert decode_kv_bytes([1, 17], 2, 64, 2) == 18 * 2 * 2 * 64 * 2
