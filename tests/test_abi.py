"""Host-side checks of the C ABI library (no GPU): it loads, exports every
function include/kvq.h declares, the Python binding covers the same names,
and the host-only calls (pool sizing, status strings) agree with the oracle's
independent layout."""
import os
import re

import pytest

import oracle as O
import quantized_kv_cache_16_b200 as K

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    txt = open(os.path.join(ROOT, "include", "kvq.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return set(re.findall(r"\b(kvq_[a-z_0-9]+)\s*\(", txt))


def test_header_declares_the_binding_names():
    assert _declared() == set(K.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = K.lib()
    for name in _declared():
        assert hasattr(L, name), name


CONFIGS = [
    dict(num_q_heads=8, num_kv_heads=2, head_dim=64),
    dict(num_q_heads=32, num_kv_heads=8, head_dim=128),
    dict(num_q_heads=8, num_kv_heads=2, head_dim=64, rotate=2),
    dict(num_q_heads=32, num_kv_heads=8, head_dim=128, k_fmt=2, v_fmt=2, k_group=128, v_group=128, rotate=2),
    dict(num_q_heads=32, num_kv_heads=8, head_dim=128, k_fmt=1, k_group=128, bound_block_tokens=128),
    dict(num_q_heads=32, num_kv_heads=8, head_dim=128, k_fmt=2, v_fmt=2, k_group=128, v_group=128, clip_ratio=0.9),
    dict(num_q_heads=64, num_kv_heads=8, head_dim=128, num_pages=3),
    dict(num_q_heads=32, num_kv_heads=8, head_dim=128, k_fmt=3, v_fmt=3, k_group=4, v_group=4),
    dict(num_q_heads=8, num_kv_heads=1, head_dim=128, k_fmt=3, v_fmt=3, k_group=4, v_group=4, num_pages=5),
    dict(num_q_heads=32, num_kv_heads=8, head_dim=128, k_fmt=4, v_fmt=4, k_group=16, v_group=16),
    dict(num_q_heads=32, num_kv_heads=8, head_dim=128, k_fmt=4, v_fmt=4, k_group=16, v_group=16, scale_search=1),
]


@pytest.mark.parametrize("kw", CONFIGS)
def test_pool_bytes_matches_oracle_layout(kw):
    kw = dict(kw)
    kw.setdefault("num_pages", 37)
    assert K.kvq_pool_bytes(K.make_config(**kw)) == O.pool_bytes(O.make_config(**kw))


@pytest.mark.parametrize("bad", [
    dict(head_dim=96), dict(num_q_heads=12, num_kv_heads=8), dict(num_q_heads=72, num_kv_heads=8),
    dict(num_pages=0), dict(k_group=64), dict(v_fmt=1, v_group=128), dict(clip_ratio=0.0),
    dict(clip_ratio=1.5), dict(bound_block_tokens=100), dict(k_fmt=7), dict(rotate=3), dict(rotate=-1),
    # HQMQ: keys and values both, group 4, head_dim 128, no descriptors or scale search
    dict(k_fmt=3, k_group=4), dict(v_fmt=3, v_group=4), dict(k_fmt=3, v_fmt=3, k_group=4, v_group=32),
    dict(k_fmt=3, v_fmt=3, k_group=4, v_group=4, head_dim=64, num_q_heads=8, num_kv_heads=2),
    dict(k_fmt=3, v_fmt=3, k_group=4, v_group=4, bound_block_tokens=64),
    dict(k_fmt=3, v_fmt=3, k_group=4, v_group=4, scale_search=1),
    dict(k_fmt=3, v_fmt=3, k_group=4, v_group=4, rotate=2),
    # NVFP4: keys and values both, group 16, head_dim 128, no descriptors
    dict(k_fmt=4, k_group=16), dict(k_fmt=4, v_fmt=4, k_group=16, v_group=32),
    dict(k_fmt=4, v_fmt=4, k_group=16, v_group=16, head_dim=64, num_q_heads=8, num_kv_heads=2),
    dict(k_fmt=4, v_fmt=4, k_group=16, v_group=16, bound_block_tokens=64),
    dict(k_fmt=4, v_fmt=4, k_group=16, v_group=16, rotate=2),
])
def test_invalid_configs_have_no_pool(bad):
    kw = dict(num_q_heads=32, num_kv_heads=8, head_dim=128, num_pages=4)
    kw.update(bad)
    assert K.kvq_pool_bytes(K.make_config(**kw)) == 0


def test_status_strings():
    assert K.kvq_status_string(K.KVQ_OK) == "ok"
    for s in range(1, 7):
        assert K.kvq_status_string(s) not in ("ok", "unknown status")
    assert K.kvq_status_string(99) == "unknown status"
