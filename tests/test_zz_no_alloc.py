"""The allocation-free Full-attention entry point against the regular one
and against the float64 oracle.

oda_full_attn_gated_static exists for callers that cannot call cudaMalloc
(engines whose device memory all belongs to their own pool allocator, decode
loops that must not synchronize the device). It keeps its scratch in fixed
device arrays inside liboda. Here it must reproduce oda_full_attn_gated on
two calls in a row -- the second reuses the arrays the first left behind --
within the attention tolerance the other tests use. This file is collected
last on purpose.
"""

import numpy as np
import pytest

import synth
from tests import _harness as hx

pytestmark = pytest.mark.gpu


def test_static_entry_point_matches_regular_twice():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from gated_local_full_b200 import oda
    w = synth.custom("noalloc", layers=2, batch=4, hq=16, hkv=8, d=128, window=256,
                     t0=(9000, 300, 4100, 17), fixed_scores=(1.0, -1.0, 1.0, 1.0))
    ctx, dw = hx.setup(w)
    B = w.batch
    seq = dw.seq_lens[0]
    for l in range(w.layers):
        ctx.append_kv(l, l + 1, dw.k_new[0, l], dw.v_new[0, l], seq, dw.block_table, dw.cache,
                      dw.ring, B)
    flags = torch.empty(B, dtype=torch.uint8, device="cuda")
    idx = torch.empty(B, dtype=torch.int32, device="cuda")
    count = torch.empty(1, dtype=torch.int32, device="cuda")
    ctx.gate(dw.scores[0], 0.0, B, flags, idx, count)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    atol, rtol = hx.tol(w)
    for call, layer in enumerate((1, 0)):         # two calls in a row
        ref = torch.zeros((B, w.hq, w.d), dtype=torch.bfloat16, device="cuda")
        ref_lse = torch.zeros((B, w.hq), dtype=torch.float32, device="cuda")
        ctx.full_attn_gated(layer, dw.q[0, layer], seq, dw.block_table, dw.cache, idx, count,
                            ref, ref_lse, B)
        got = torch.zeros_like(ref)
        got_lse = torch.zeros_like(ref_lse)
        oda.full_attn_gated_static(ctx.cfg, layer, dw.q[0, layer], seq, dw.block_table,
                                   dw.cache, idx, count, got, got_lse, B, err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0 and ctx.get_device_error() == 0
        hx.assert_close(got.to(torch.float64).cpu().numpy(), ref.to(torch.float64).cpu().numpy(),
                        atol, rtol, f"call {call} out")
        hx.assert_close(got_lse.cpu().numpy().astype(np.float64),
                        ref_lse.cpu().numpy().astype(np.float64), 1e-4, 1e-5, f"call {call} lse")
        # unflagged row 1 is left untouched by both
        assert torch.count_nonzero(got[1]) == 0
        # and the flagged rows equal the float64 oracle's Full attention
        g64 = got.to(torch.float64).cpu().numpy()
        for r in (0, 2, 3):
            want = hx.oracle_row(w, 0, layer, r)
            hx.assert_close(g64[r], want["full"], atol, rtol, f"call {call} row {r} vs oracle")
            hx.assert_close(got_lse[r].cpu().numpy().astype(np.float64), want["lse_full"],
                            1e-4, 1e-5, f"call {call} row {r} lse vs oracle")
    # sizes beyond the fixed arrays are refused before any launch
    big = oda.make_config(layers=1, max_batch=128, hq=16, hkv=8, head_dim=128, sink=4,
                          window=256, dtype="bf16", max_blocks_per_seq=dw.max_blocks,
                          num_blocks=dw.num_blocks)
    with pytest.raises(oda.OdaError) as e:
        oda.full_attn_gated_static(big, 0, dw.q[0, 0], seq, dw.block_table, dw.cache, idx,
                                   count, got, None, 128)
    assert e.value.status == oda.ERR_SHAPE
