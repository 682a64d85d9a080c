"""The decode split plan, read back through the workspace-size query on the
host (no GPU): every (sequence, KV head) unit is cut into splits of a chunk of
whole 256-token tiles, the chunk chosen so that the full items fill a whole
number of rounds of the resident CTAs (two per SM on 148 SMs). The pinned
cases are the workloads whose timings chose the rule."""
import ctypes

import pytest

from bit_kv_cache_21_b200 import build as kbuild

FAKE = 0x100000  # 16-byte aligned, never dereferenced by the host query
ROW_BYTES = 128 * 4 + 8  # one partial: o row and (m, l)


@pytest.fixture(scope="module")
def K():
    kbuild.build()
    import bit_kv_cache_21_b200 as K
    return K


def _desc(K, **kw):
    d = dict(num_seqs=16, num_kv_heads=8, head_dim=128, bits_k=4, bits_v=4, group_k=128, group_v=128,
             axis_k=0, axis_v=0, hadamard_block_k=128, residual_len=0, paged=0, page_size=0,
             max_pages_per_seq=0, num_pages=0, capacity_tokens=8320, reserved=0, k_codes=FAKE,
             v_codes=FAKE, k_sz=FAKE, v_sz=FAKE, k_res=None, v_res=None, block_table=None, status=None)
    d.update(kw)
    return K.CacheDesc(**d)


def _n_split(K, desc, num_seqs, num_q_heads, max_seq_len):
    ws = int(K.lib().kvq_decode_workspace_size(ctypes.byref(desc), num_seqs, num_q_heads, max_seq_len))
    rows = num_seqs * num_q_heads
    assert ws > 16 and (ws - 16) % (rows * ROW_BYTES) == 0, ws
    return (ws - 16) // (rows * ROW_BYTES)


def test_llama8b_layer_takes_1024_token_splits(K):
    # 128 units of 8256 tokens: 8 full 1024-token splits (3.46 items per
    # resident CTA) and a 64-token trailing split, the smallest tail of the
    # equally even choices
    d = _desc(K)
    assert _n_split(K, d, 16, 32, 8256) == 9
    assert _n_split(K, d, 16, 32, 8320) == 9


def test_long_int2_takes_1792_token_splits(K):
    # 8 units of 131072 tokens: 73 full 1792-token splits = 584 items, 1.97 per
    # resident CTA, and a 256-token trailing split
    d = _desc(K, num_seqs=1, bits_k=2, bits_v=2, axis_k=1, group_k=128, group_v=32, hadamard_block_k=0,
              residual_len=128, capacity_tokens=131072 + 128, k_res=FAKE, v_res=FAKE)
    assert _n_split(K, d, 1, 32, 131072) == 74


def test_many_units_take_the_longest_chunk(K):
    # 512 units up to 32772 tokens (paged_mix): more work than 4.5 items per
    # CTA at any chunk, so the longest one, 2048 tokens
    d = _desc(K, num_seqs=64, paged=1, page_size=16, max_pages_per_seq=2049, num_pages=1 << 17,
              block_table=FAKE, capacity_tokens=0)
    assert _n_split(K, d, 64, 32, 32772) == 17


def test_little_work_takes_one_tile_per_split(K):
    d = _desc(K, num_seqs=1, num_kv_heads=1, capacity_tokens=1024)
    assert _n_split(K, d, 1, 4, 256) == 1
    assert _n_split(K, d, 1, 4, 1000) == 4
    assert _n_split(K, d, 1, 4, 0) == 1  # the workspace still holds one split


def test_bf16_caches_keep_eight_items_per_sm(K):
    # attention over rematerialized bf16 K/V (one CTA per SM): 64 units of 16384
    # tokens in 1024-token chunks
    d = _desc(K, num_seqs=8, bits_k=16, bits_v=16, hadamard_block_k=0, capacity_tokens=16384,
              k_sz=None, v_sz=None)
    assert _n_split(K, d, 8, 32, 16384) == 16


@pytest.mark.parametrize("max_seq_len", [1, 255, 257, 4097, 65537, 1 << 20, (1 << 31) - 1])
def test_split_count_is_bounded(K, max_seq_len):
    d = _desc(K, num_seqs=2, num_kv_heads=2, capacity_tokens=1024)
    n = _n_split(K, d, 2, 8, max_seq_len)
    assert 1 <= n <= 512
    # a split is 1 to max(8, ceil(L / 512 tiles)) tiles long
    tiles = -(-max_seq_len // 256)
    longest = max(8, -(-tiles // 512))
    assert -(-tiles // longest) <= n <= tiles
