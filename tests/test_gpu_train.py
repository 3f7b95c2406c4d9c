"""GPU parity of the recall head's training objective (oda_recall_loss)
against the float64 oracle: mean Huber_1(q - T(g - lambda)) and the count of
positions whose access gain g = log p^F - log p^L exceeds lambda.

Both sides form the gain f - l and compare it with lambda in float64 from the
float32 inputs, so the count is compared bit-exactly; the loss (the device
takes T's logarithm in float32) within 1e-6 + 1e-5 relative."""

import numpy as np
import pytest

import oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch as _t
    if not _t.cuda.is_available():
        pytest.skip("needs a GPU")
    return _t


@pytest.fixture(scope="module")
def ctx(torch):
    from gated_local_full_b200 import oda
    cfg = oda.make_config(layers=1, max_batch=1, hq=2, hkv=1, head_dim=64, sink=4, window=16,
                          dtype="f32", max_blocks_per_seq=4, num_blocks=4)
    c = oda.OdaContext(cfg)
    yield c
    c.close()


def _inputs(n, seed, lam):
    rng = np.random.default_rng(seed)
    q = rng.normal(0.0, 2.0, n).astype(np.float32)                 # head outputs
    lf = rng.normal(-2.0, 1.5, n).astype(np.float32)               # log p^F
    ll = (lf - rng.normal(0.1, 1.0, n)).astype(np.float32)         # log p^L
    k = n // 7
    lf[:k] = np.float32(lam)                                        # ties: g == lambda exactly
    ll[:k] = np.float32(0.0)
    return q, lf, ll


def _oracle(q, lf, ll, lam):
    g = O.access_gain(lf, ll)                                       # float64, as the device
    y = O.regression_target(g, float(lam))
    return O.recall_regression_loss(q, y), int(O.best_action(g, float(lam)).sum())


@pytest.mark.parametrize("n", [1, 7, 1000, 1 << 20, (1 << 20) + 3])
@pytest.mark.parametrize("lam", [0.0, 0.25, -1.5])
def test_recall_loss_matches_oracle(torch, ctx, n, lam):
    q, lf, ll = _inputs(n, n * 31 + int(lam * 8), lam)
    loss = torch.zeros(1, dtype=torch.float32, device="cuda")
    nf = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq, dlf, dll = (torch.from_numpy(a).cuda() for a in (q, lf, ll))
    ctx.recall_loss(dq, dlf, dll, lam, loss, nf)
    torch.cuda.synchronize()
    assert ctx.get_device_error() == 0
    ref_loss, ref_count = _oracle(q, lf, ll, np.float32(lam))
    assert int(nf.item()) == ref_count
    got = float(loss.item())
    assert abs(got - ref_loss) <= 1e-6 + 1e-5 * abs(ref_loss), (got, ref_loss)
    # the same call again gives the same bits (fixed-order reduction)
    loss2 = torch.zeros_like(loss)
    ctx.recall_loss(dq, dlf, dll, lam, loss2, nf)
    torch.cuda.synchronize()
    assert torch.equal(loss, loss2)


def test_recall_loss_closed_forms(torch, ctx):
    """q = y exactly gives loss 0; one position with r = 3 gives 3 - 1/2;
    one with r = 0.5 gives 0.125."""
    f = lambda a: torch.tensor(a, dtype=torch.float32, device="cuda")
    loss = torch.zeros(1, dtype=torch.float32, device="cuda")
    nf = torch.zeros(1, dtype=torch.int32, device="cuda")
    # g = 0 - 0 = 0, lambda = 0: y = T(0) = 0
    ctx.recall_loss(f([0.0]), f([0.0]), f([0.0]), 0.0, loss, nf)
    torch.cuda.synchronize()
    assert float(loss.item()) == 0.0 and int(nf.item()) == 0
    ctx.recall_loss(f([3.0]), f([0.0]), f([0.0]), 0.0, loss, nf)
    torch.cuda.synchronize()
    assert float(loss.item()) == 2.5
    ctx.recall_loss(f([0.5]), f([0.0]), f([0.0]), 0.0, loss, nf)
    torch.cuda.synchronize()
    assert float(loss.item()) == 0.125


def test_recall_loss_rejects_bad_arguments(torch, ctx):
    from gated_local_full_b200 import oda
    loss = torch.zeros(1, dtype=torch.float32, device="cuda")
    nf = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = oda.lib().oda_recall_loss(ctx.handle, None, None, None, 0.0, 0, oda.ptr(loss),
                                   oda.ptr(nf), None)
    assert st == oda.ERR_ARG
