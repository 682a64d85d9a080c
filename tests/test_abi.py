"""The C-ABI library loads, exports every symbol include/kvq.h declares, and
rejects bad arguments on the host without launching anything (no GPU needed)."""
import ctypes
import subprocess

import pytest

from bit_kv_cache_21_b200 import build as kbuild

FAKE = 0x100000  # 16-byte aligned, never dereferenced by host validation


@pytest.fixture(scope="module")
def K():
    kbuild.build()
    import bit_kv_cache_21_b200 as K
    return K


def _desc(K, **kw):
    d = dict(num_seqs=2, num_kv_heads=8, head_dim=128, bits_k=4, bits_v=4, group_k=128,
             group_v=128, axis_k=0, axis_v=0, hadamard_block_k=128, residual_len=0, paged=0,
             page_size=0, max_pages_per_seq=0, num_pages=0, capacity_tokens=1024, reserved=0,
             k_codes=FAKE, v_codes=FAKE, k_sz=FAKE, v_sz=FAKE, k_res=None, v_res=None,
             block_table=None, status=None)
    d.update(kw)
    return K.CacheDesc(**d)


def test_library_exports_every_declared_symbol(K):
    names = K.header_symbols()
    assert set(names) >= {"kvq_quantize_append", "kvq_decode_attention", "kvq_remat_kv",
                          "kvq_decode_workspace_size", "kvq_decode_splitk", "kvq_decode_merge",
                          "kvq_rope_tables", "kvq_status_string", "kvq_debug_set", "kvq_version"}
    out = subprocess.run(["nm", "-D", "--defined-only", kbuild.LIB], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    for n in names:
        assert n in exported, n
        assert hasattr(K.lib(), n)
    # nothing else of ours leaks out of the library
    assert {n for n in exported if n.startswith("kvq")} == set(names)


def test_status_strings_and_version(K):
    assert K.status_string(K.OK) == "ok"
    assert "invalid" in K.status_string(K.ERR_INVALID_ARG)
    assert K.version() >= 100


def _append(K, d, dtype=0, total=4, v_new=FAKE):
    return K.lib().kvq_quantize_append(ctypes.byref(d) if d is not None else None, FAKE, v_new,
                                       dtype, FAKE, FAKE, 2, total, None)


def test_append_validation(K):
    E, U = K.ERR_INVALID_ARG, K.ERR_UNSUPPORTED
    assert _append(K, None) == E
    assert _append(K, _desc(K, head_dim=64)) == U
    assert _append(K, _desc(K, bits_k=3)) == E
    assert _append(K, _desc(K, group_k=24)) == E
    assert _append(K, _desc(K, hadamard_block_k=96)) == E
    assert _append(K, _desc(K, k_codes=FAKE + 4)) == E
    assert _append(K, _desc(K, capacity_tokens=1000)) == E
    assert _append(K, _desc(K, reserved=1)) == E
    assert _append(K, _desc(K, hybrid=2)) == E          # hybrid is 0 or 1
    # randomized-Hadamard signs need a rotation and 16-byte alignment
    assert _append(K, _desc(K, hadamard_block_k=0, hadamard_signs=FAKE)) == E
    assert _append(K, _desc(K, hadamard_signs=FAKE + 4)) == E
    assert _append(K, _desc(K), dtype=7) == E
    assert _append(K, _desc(K), v_new=None) == E          # V cache but no V input
    # values grouped along tokens: per channel over the window's blocks only
    assert _append(K, _desc(K, axis_v=2)) == E
    assert _append(K, _desc(K, axis_v=1)) == U                               # rotation
    assert _append(K, _desc(K, axis_v=1, hadamard_block_k=0)) == E           # no window
    chan_v = dict(axis_v=1, bits_k=2, bits_v=2, group_k=128, group_v=128, hadamard_block_k=0,
                  residual_len=128, k_res=FAKE, v_res=FAKE)
    assert _append(K, _desc(K, **dict(chan_v, group_v=64))) == E             # group != window
    assert _append(K, _desc(K, **dict(chan_v, bits_v=4))) == U               # mixed widths
    # per-channel keys need the residual window and a contiguous cache
    assert _append(K, _desc(K, axis_k=1, hadamard_block_k=0, residual_len=0)) == E
    assert _append(K, _desc(K, axis_k=1, hadamard_block_k=0, residual_len=128, paged=1,
                            page_size=16, max_pages_per_seq=4, num_pages=8, block_table=FAKE)) == U
    # the window needs bf16 appends and no rotation
    kivi = dict(axis_k=1, bits_k=2, bits_v=2, group_k=128, group_v=32, hadamard_block_k=0,
                residual_len=128, k_res=FAKE, v_res=FAKE)
    assert _append(K, _desc(K, **kivi), dtype=K.FP32) == U
    assert _append(K, _desc(K, **dict(kivi, hadamard_block_k=128))) == U
    # paged needs a page size, pool and block table
    assert _append(K, _desc(K, paged=1, page_size=12, max_pages_per_seq=4, num_pages=8,
                            block_table=FAKE)) == E
    assert _append(K, _desc(K, paged=1, page_size=16, max_pages_per_seq=4, num_pages=8,
                            block_table=None)) == E
    # bf16 caches are written by rematerialization, not appended
    assert _append(K, _desc(K, bits_k=16, bits_v=16, hadamard_block_k=0)) == U


def _decode(K, d, hq=32, ws=1 << 30, max_len=512, out=FAKE, q_dtype=0, scale=0.088):
    return K.lib().kvq_decode_attention(ctypes.byref(d), FAKE, q_dtype, hq, FAKE, 2, max_len,
                                        scale, out, FAKE, ws, None)


def test_decode_validation(K):
    d = _desc(K)
    assert _decode(K, d, hq=20) == K.ERR_INVALID_ARG         # not a multiple of H
    assert _decode(K, d, hq=24) == K.ERR_UNSUPPORTED         # GQA 3
    assert _decode(K, d, hq=64) == K.ERR_UNSUPPORTED         # GQA 8
    assert _decode(K, d, out=None) == K.ERR_INVALID_ARG
    assert _decode(K, d, max_len=2048) == K.ERR_INVALID_ARG  # beyond capacity
    assert _decode(K, d, ws=16) == K.ERR_CAPACITY            # workspace too small
    assert _decode(K, d, q_dtype=9) == K.ERR_INVALID_ARG
    assert _decode(K, d, scale=float("nan")) == K.ERR_INVALID_ARG


def test_partial_merge_validation(K):
    d = _desc(K)
    mp = K.lib().kvq_decode_merge_partial
    ws = K.decode_workspace_size(d, 2, 32, 512)
    assert mp(ctypes.byref(d), 32, FAKE, 2, 512, None, FAKE, FAKE, ws, None) == K.ERR_INVALID_ARG
    assert mp(ctypes.byref(d), 32, FAKE, 2, 512, FAKE, FAKE + 4, FAKE, ws, None) == K.ERR_INVALID_ARG
    assert mp(ctypes.byref(d), 32, FAKE, 2, 512, FAKE, FAKE, FAKE, 16, None) == K.ERR_CAPACITY
    assert mp(ctypes.byref(d), 0, FAKE, 2, 512, FAKE, FAKE, FAKE, ws, None) == K.ERR_INVALID_ARG
    mg = K.lib().kvq_merge_partials
    assert mg(None, 2, 2, 32, FAKE, None) == K.ERR_INVALID_ARG
    assert mg(FAKE + 8, 2, 2, 32, FAKE, None) == K.ERR_INVALID_ARG         # parts not 16-byte aligned
    assert mg(FAKE, 0, 2, 32, FAKE, None) == K.ERR_INVALID_ARG
    assert mg(FAKE, 2, 70000, 32, FAKE, None) == K.ERR_INVALID_ARG         # grid limit on sequences
    assert mg(FAKE, 2, 2, 32, None, None) == K.ERR_INVALID_ARG


def test_workspace_size(K):
    d = _desc(K)
    ws = K.decode_workspace_size(d, 2, 32, 512)
    # partial outputs and (max, sum) pairs per (sequence, query head, split), plus a counter
    assert ws > 16 and (ws - 16) % (2 * 32 * (128 * 4 + 8)) == 0
    assert K.decode_workspace_size(d, 2, 32, 8192) >= ws
    assert K.decode_workspace_size(d, 0, 32, 512) == 0


def test_remat_and_rope_validation(K):
    x = _desc(K, num_kv_heads=32, hadamard_block_k=0, v_codes=None, v_sz=None, bits_v=0)
    call = K.lib().kvq_remat_kv
    assert call(ctypes.byref(x), FAKE, 8, FAKE, FAKE, 2, 100, FAKE, FAKE, None) == K.ERR_INVALID_ARG
    assert call(ctypes.byref(_desc(K, num_kv_heads=32, hadamard_block_k=128, v_codes=None)),
                FAKE, 8, FAKE, FAKE, 2, 128, FAKE, FAKE, None) == K.ERR_UNSUPPORTED
    assert call(ctypes.byref(x), None, 8, FAKE, FAKE, 2, 128, FAKE, FAKE, None) == K.ERR_INVALID_ARG
    fused = K.lib().kvq_remat_attention
    ws = K.lib().kvq_remat_attention_workspace_size(2, 32, 1024)
    assert ws == 2 * 32 * 8 * (128 * 4 + 8)
    assert K.lib().kvq_remat_attention_workspace_size(2, 32, 1000) == 0
    args = lambda **kw: [kw.get(n, d) for n, d in (("w", FAKE), ("h", 8), ("c", FAKE), ("s", FAKE), ("b", 2),
                                                  ("t", 1024), ("q", FAKE), ("qd", 0), ("hq", 32),
                                                  ("sc", 0.088), ("o", FAKE), ("ws", FAKE), ("wb", ws))]
    xb = _desc(K, num_kv_heads=32, hadamard_block_k=0, v_codes=None, v_sz=None, bits_v=0, capacity_tokens=1024)
    assert fused(ctypes.byref(xb), *args(t=1000), None) == K.ERR_INVALID_ARG        # not whole tiles
    assert fused(ctypes.byref(xb), *args(hq=24), None) == K.ERR_UNSUPPORTED         # GQA 3
    assert fused(ctypes.byref(xb), *args(hq=30), None) == K.ERR_INVALID_ARG         # not a multiple
    assert fused(ctypes.byref(xb), *args(q=None), None) == K.ERR_INVALID_ARG
    assert fused(ctypes.byref(xb), *args(qd=7), None) == K.ERR_INVALID_ARG
    assert fused(ctypes.byref(xb), *args(wb=ws - 1), None) == K.ERR_CAPACITY
    assert K.lib().kvq_rope_tables(FAKE, FAKE, 0, 128, 500000.0, None) == K.ERR_INVALID_ARG
    assert K.lib().kvq_rope_tables(FAKE, FAKE, 16, 127, 500000.0, None) == K.ERR_INVALID_ARG


def test_debug_hooks_validation(K):
    assert K.lib().kvq_debug_set(99, 0) == K.ERR_INVALID_ARG
    assert K.lib().kvq_debug_set(K.DEBUG_SKIP_TILE, -1) == K.OK
    assert K.lib().kvq_debug_set(K.DEBUG_WAIT_TIMEOUT_NS, 0) == K.OK
