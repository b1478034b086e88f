"""The C ABI library on the host: it loads without a GPU, exports every function that
include/hymba.h declares, and its host-only logic (workspace sizing, stage layout, KV
sharing plan, argument validation) behaves as documented."""
import ctypes

import numpy as np
import pytest

from hybrid_attention_ssm_b200 import build as hbuild
from hybrid_attention_ssm_b200 import hymba as H
from hybrid_attention_ssm_b200 import synth
from oracle import hymba_oracle as orc


@pytest.fixture(scope="module", autouse=True)
def _lib():
    hbuild.build()
    H.lib()


def test_exports_every_declared_function():
    names = H.header_functions()
    assert len(names) >= 14
    L = ctypes.CDLL(H.LIB_PATH)
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/hymba.h but not exported"
    assert H.lib().hymba_version() >= 10000


def test_workspace_sizes_grow_with_tokens():
    d = synth.workloads()["swa"].dims
    a = H.workspace_size(d, 1, 2048)
    b = H.workspace_size(d, 1, 4096)
    assert 0 < a < b
    lay = H.stage_layout(d, 1, 2048)
    offs = [lay.q, lay.xz, lay.xc, lay.xbc, lay.dt_pre, lay.y, lay.o, lay.u]
    assert all(o % 256 == 0 for o in offs) and offs == sorted(offs) and offs[-1] < a
    assert lay.ld_xbc >= 132
    assert lay.scan_chunks >= 1 and lay.scan_chunk_len % 8 == 0
    assert lay.scan_chunks * lay.scan_chunk_len >= 2176 > (lay.scan_chunks - 1) * lay.scan_chunk_len


@pytest.mark.parametrize("B,N,Di", [(1, 2048, 3200), (4, 8192, 3200), (8, 4096, 3200), (1, 120, 512),
                                    (3, 1, 512), (64, 100, 3200), (2, 37, 64)])
def test_scan_chunking_matches_bench_accounting(B, N, Di):
    """bench.py counts the scan's bytes per chunk the way the library cuts T into chunks."""
    import bench
    d = synth.workloads()["tiny"].dims.replace(d_inner=Di, n_meta=8)
    lay = H.stage_layout(d, B, N)
    T = 8 + N
    assert bench.scan_chunks(B, Di, T) == (lay.scan_chunk_len, lay.scan_chunks)
    assert (lay.scan_chunks - 1) * lay.scan_chunk_len < T <= lay.scan_chunks * lay.scan_chunk_len
    dec = H.workspace_size(d, 64, 0, 0, H.MODE_DECODE)
    assert dec > 0


@pytest.mark.parametrize("T,M,W,is_global", [(2176, 128, 1024, 0), (300, 8, 32, 1), (270, 130, 100, 0),
                                               (308, 8, 1, 0), (140, 0, 64, 0)])
def test_bench_visible_pairs_equal_the_oracle_mask(T, M, W, is_global):
    """The attention FLOPs in bench.py's roofline count the (query, key) pairs the oracle's
    visibility mask allows (the SWA layer: 1,843,776 per head)."""
    import bench
    pos = np.arange(T)
    assert bench.visible_pairs(T, M, W, is_global) == int(orc.visibility_mask(pos, pos, M, W, is_global).sum())
    if (T, M, W) == (2176, 128, 1024):
        assert bench.visible_pairs(T, M, W, is_global) == 1843776


@pytest.mark.parametrize("field,value,code", [("head_dim", 32, H.ERR_UNSUPPORTED),
                                              ("d_state", 8, H.ERR_UNSUPPORTED),
                                              ("d_inner", 100, H.ERR_UNSUPPORTED),
                                              ("n_kv_heads", 3, H.ERR_UNSUPPORTED),
                                              ("dt_rank", 6, H.ERR_UNSUPPORTED),
                                              ("window", 0, H.ERR_INVALID_ARG),
                                              ("kv_role", 7, H.ERR_INVALID_ARG)])
def test_invalid_configs_are_rejected(field, value, code):
    d = synth.workloads()["tiny"].dims.replace(**{field: value})
    with pytest.raises(H.HymbaError) as e:
        H.workspace_size(d, 1, 16)
    assert e.value.code == code


def test_size_limits_are_accepted_and_one_step_beyond_rejected():
    """The widest configuration the kernels take (the GPU parity suite runs it) passes the
    host checks; one step past any of its limits is refused before anything launches."""
    lim = synth.workloads()["tiny"].dims.replace(d_model=1024, n_q_heads=32, n_kv_heads=8, d_inner=4096,
                                                 dt_rank=224, n_meta=8, window=48)
    assert H.workspace_size(lim, 2, 60) > 0
    assert H.workspace_size(lim, 2, 69, 0, H.MODE_DECODE) > 0
    for kw in (dict(d_inner=4096 + 64), dict(n_q_heads=33, n_kv_heads=11), dict(dt_rank=228),
               dict(n_q_heads=28, n_kv_heads=4)):
        with pytest.raises(H.HymbaError) as e:
            H.workspace_size(lim.replace(**kw), 2, 60)
        assert e.value.code == H.ERR_UNSUPPORTED, kw


def test_kv_share_plan_matches_oracle_reading():
    d = synth.workloads()["stack"].dims
    is_global = [1 if i in (0, 15, 31) else 0 for i in range(32)]
    need, cid, role, caches = H.kv_share_alloc(d, is_global, 8, 4224)
    ocid, orole = orc.kv_share_plan(is_global)
    assert cid == ocid and role == orole
    assert len(caches) == 18
    row = d.n_kv_heads * d.head_dim * 2
    full = 8 * 4224 * row
    swa = 2 * (8 * d.n_meta * row + 8 * d.window * row)
    assert need == 2 * full + 3 * 2 * full + 15 * swa      # view + 3 global + 15 SWA caches


def test_kv_share_odd_patterns():
    d = synth.workloads()["tiny"].dims
    for pattern in ([0], [1], [0, 0, 0], [0, 1, 0, 0, 1], [1, 1, 1]):
        need, cid, role, _ = H.kv_share_alloc(d, pattern, 1, 64)
        ocid, orole = orc.kv_share_plan(pattern)
        assert (cid, role) == (ocid, orole), pattern
        assert need > 0


def test_l2_prefetch_arguments_are_checked_on_the_host():
    """hymba_l2_prefetch refuses 0 or more than 8 ranges and null or misaligned pointers
    before it launches anything."""
    L = H.lib()
    ptrs = (ctypes.c_void_p * 9)(*([256] * 9))
    sizes = (ctypes.c_size_t * 9)(*([4096] * 9))
    for n in (0, 9):
        assert L.hymba_l2_prefetch(ptrs, sizes, n, None) == H.ERR_INVALID_ARG
    bad = (ctypes.c_void_p * 1)(None)
    assert L.hymba_l2_prefetch(bad, sizes, 1, None) == H.ERR_INVALID_ARG
    odd = (ctypes.c_void_p * 1)(264)
    assert L.hymba_l2_prefetch(odd, sizes, 1, None) == H.ERR_INVALID_ARG


def test_ffn_decode_workspace_sizes():
    """The decode FFN's workspace holds its split-K slices and activations: it grows with the
    rows, and shapes outside the kernels' limits are refused."""
    a = H.ffn_workspace_size(1, 1600, 5504)
    b = H.ffn_workspace_size(8, 1600, 5504)
    c = H.ffn_workspace_size(64, 1600, 5504)
    assert 0 < a < b < c
    assert c >= 64 * 5504 * 2 + 64 * 1600 * 4   # fp16 activations and at least one fp32 slice
    for rows, d, F in ((0, 1600, 5504), (257, 1600, 5504), (8, 1602, 5504), (8, 1600, 5500)):
        with pytest.raises(H.HymbaError) as e:
            H.ffn_workspace_size(rows, d, F)
        assert e.value.code == H.ERR_INVALID_ARG
