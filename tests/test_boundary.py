"""CPU checks of the C ABI: the library loads, exports every declared symbol,
and validates arguments before touching the GPU (no compute calls here)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "oda.h")


def _ensure_built():
    from gated_local_full_b200 import oda
    from synth import device
    if not (os.path.exists(oda.LIB_PATH) and os.path.exists(device.LIB_PATH)):
        from gated_local_full_b200.build import build
        build()


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(oda_[a-z_0-9]+)\s*\(", src)))


def test_header_and_binding_agree():
    from gated_local_full_b200 import oda
    assert _declared() == sorted(oda.EXPORTS)


def test_library_exports_every_declared_symbol():
    _ensure_built()
    from gated_local_full_b200 import oda
    L = ctypes.CDLL(oda.LIB_PATH)
    for name in _declared():
        assert hasattr(L, name), name
    assert oda.version().startswith("oda-b200")


def test_synth_library_exports():
    _ensure_built()
    from synth import device
    L = device.lib()
    assert hasattr(L, "synth_fill_streams") and hasattr(L, "synth_fill_paged_kv")


def _cfg(**over):
    from gated_local_full_b200 import oda
    base = dict(layers=28, max_batch=8, hq=16, hkv=8, head_dim=128, sink=4, window=2048,
                dtype="bf16", max_blocks_per_seq=8257, num_blocks=8257)
    base.update(over)
    return oda.make_config(**base)


def test_layout_values():
    _ensure_built()
    from gated_local_full_b200 import oda
    lay = oda.layout(_cfg())
    assert lay["elem_bytes"] == 2
    assert lay["tile_elems"] == 2 * 16 * 128
    assert lay["ring_blocks"] == 129                     # ceil(2052 / 16)
    assert lay["cache_layer_elems"] == 8257 * 8 * 4096
    assert lay["ring_layer_elems"] == 8 * 8 * 129 * 4096
    assert oda.layout(_cfg(dtype="f32"))["elem_bytes"] == 4


@pytest.mark.parametrize("over,code", [
    (dict(head_dim=96), 2), (dict(hq=12, hkv=8), 2), (dict(hq=24, hkv=3), 2),
    (dict(block_size=32), 2), (dict(max_batch=1025), 2), (dict(dtype=7), 3),
    (dict(layers=0), 1), (dict(window=0), 1), (dict(sink=-1), 1), (dict(num_blocks=0), 1),
    (dict(max_batch=1024, max_blocks_per_seq=1 << 20), 2),
])
def test_layout_rejects_bad_configs(over, code):
    _ensure_built()
    from gated_local_full_b200 import oda
    with pytest.raises(oda.OdaError) as e:
        oda.layout(_cfg(**over))
    assert e.value.status == code


def test_null_context_and_pointers_rejected_without_gpu():
    _ensure_built()
    from gated_local_full_b200 import oda
    L = oda.lib()
    assert L.oda_layout(None, None) == oda.ERR_ARG
    assert L.oda_create(None, None) == oda.ERR_ARG
    assert L.oda_destroy(None) == oda.OK
    assert L.oda_append_kv(None, 0, 1, None, None, None, None, None, None, 1, None) == oda.ERR_ARG
    assert L.oda_local_attn(None, 0, None, None, None, None, None, 1, 0, None) == oda.ERR_ARG
    assert L.oda_full_attn_gated(None, 0, None, None, None, None, None, None, None, None, 1, 0,
                                 None) == oda.ERR_ARG
    assert L.oda_gate(None, None, 0.0, 1, None, None, None, None) == oda.ERR_ARG
    assert L.oda_recall_score(None, None, None, None, 64, None, None, None, 0.0, 128, None, 1,
                              None) == oda.ERR_ARG
    assert L.oda_get_device_error(None, None, None) == oda.ERR_ARG
    assert L.oda_step_run(None, None, None) == oda.ERR_ARG
    assert L.oda_step_graph_launch(None, None) == oda.ERR_ARG
    assert L.oda_step_graph_destroy(None) == oda.OK
    assert L.oda_selftest_wait_timeout(None, 1000, None) == oda.ERR_ARG


def test_product_never_imports_oracle():
    """The CUDA path and the oracle share no code and neither imports the other."""
    pkg = os.path.join(ROOT, "gated_local_full_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"\boracle\b\s*(import|\.)|from\s+oracle|import\s+oracle",
                                     txt), f
    for dirpath, _, files in os.walk(os.path.join(ROOT, "oracle")):
        for f in files:
            if f.endswith(".py"):
                txt = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+(gated_local_full_b200|synth)\b", txt,
                                     flags=re.M), f
