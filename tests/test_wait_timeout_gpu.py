"""Failure detection on the GPU without a fault: the bounded mbarrier wait
that every wait in the attention kernel uses is driven to its limit by a wait
that nobody satisfies, and must end, report MXATTN_ERR_TIMEOUT and leave the
context usable for the next forward."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

TIMEOUT = 4  # MXATTN_ERR_TIMEOUT


@pytest.fixture(scope="module")
def mx():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import mxfp4_microscaled_quantization_b200 as mx

    return mx


def run_selftest(mx, arrive, timeout_us):
    out = torch.full((3,), -1, dtype=torch.int32, device="cuda")
    mx.mxattn_wait_selftest(arrive, timeout_us, out)
    torch.cuda.synchronize()
    return [int(x) for x in out.cpu()]


def test_satisfied_wait_completes(mx):
    status, waited_us, flags = run_selftest(mx, True, 1000)
    assert status == 0
    assert flags == 0
    assert waited_us < 1000


@pytest.mark.parametrize("timeout_us", [200, 2000, 20000])
def test_unsatisfied_wait_gives_up_at_its_limit(mx, timeout_us):
    status, waited_us, flags = run_selftest(mx, False, timeout_us)
    assert status == TIMEOUT
    assert flags == 3  # abort flag raised, wait left without completion
    assert waited_us >= timeout_us
    assert waited_us < timeout_us + 5000  # checked every 64 polls: ends soon after the limit


def test_context_usable_after_timeout(mx):
    run_selftest(mx, False, 500)
    from oracle import attention as oracle_attention

    w = mx.workloads.WORKLOADS["tiny"]
    Q, K, V = mx.workloads.make_qkv(w, seed=3)
    dev = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)  # noqa: E731
    q, k, v = dev(Q), dev(K), dev(V)
    O = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32, device="cuda")
    ws = mx.new_workspace(w.B, w.H, w.N, w.d)
    mx.mxattn_forward(q, k, v, w.kv_tile, True, "uos", 0.0, O, ws)
    assert mx.mxattn_workspace_status(ws) == 0
    ref = oracle_attention(Q, K, V, kv_tile=w.kv_tile, rule="uos", pnq=True)
    got = O.double().cpu().numpy()
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-3


def test_selftest_rejects_bad_arguments(mx):
    out = torch.zeros(3, dtype=torch.int32, device="cuda")
    for t in (0, 1000001):
        with pytest.raises(mx.MxattnError):
            mx.mxattn_wait_selftest(False, t, out)
