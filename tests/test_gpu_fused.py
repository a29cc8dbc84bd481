"""The single-launch decode kernel (batch <= 16) through the C ABI.

The layer forward of "Addition is almost all you need" (gist.science technical
summary, section 2.1, computation process) against the fp64 oracle, on the
cases that separate this path from the others:

* the ends of the fp16 range: x (.) b above 65504 or in the fp16 subnormal
  range, and mid (.) t above 65504.  This path keeps x (.) b and V in block
  fixed point with 22-bit magnitudes (fp32-faithful), so it matches the oracle
  in all three; the tensor-core path folds b into the sign tile exactly but
  rounds V to fp16; the two-launch decode rounds both x (.) b and V to fp16;
* a bounded device wait that runs out (a test-only flag makes rank 0 of each
  cluster wait for bytes nobody sends): the call returns, the workspace status
  word reads DBF_ERR_TIMEOUT, and after the workspace is zeroed the next call
  is correct;
* determinism (fixed reduction order) and chunks of 16 tokens.
"""
import numpy as np
import pytest
import torch

import dbf_inputs as gen
import oracle
from test_gpu_parity import PATHS, Layer, assert_fp16_close, dev, random_layer

pytestmark = pytest.mark.gpu

DBF_ERR_TIMEOUT = 6
TEST_LOSE_ARRIVAL = 1 << 30


@pytest.fixture(scope="module")
def dbf():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from binary_factorized_weight_b200 import build

    build.build()
    import binary_factorized_weight_b200 as mod

    mod.load_library()
    return mod


def _edge_layer(dbf, case, batch=3, seed=5):
    n, k, m_in = 256, 256, 512
    rng = np.random.default_rng(seed)
    A, B = gen.sign_matrix(rng, n, k), gen.sign_matrix(rng, k, m_in)
    x = gen.normal_activations(rng, batch, m_in)
    ones = np.ones
    if case == "x_b_overflows_fp16":
        # |x b| up to 4 * 60000 > 65504; V and y stay in range
        x = (x.astype(np.float64) * 20000).clip(-60000, 60000).astype(np.float16)
        b = np.full(m_in, 4.0, np.float16)
        mid = np.full(k, 2.0 ** -10, np.float16)
        a = np.full(n, 2.0 ** -10, np.float16)
    elif case == "x_b_subnormal_fp16":
        # |x b| ~ 2^-20, below the smallest normal fp16 (2^-14)
        x = (x.astype(np.float64) * 2.0 ** -10).astype(np.float16)
        b = np.full(m_in, 2.0 ** -10, np.float16)
        mid = np.full(k, 2.0 ** 10, np.float16)
        a = ones(n, np.float16)
    elif case == "mid_t_overflows_fp16":
        # |t| ~ 22, mid = 4096: |V| ~ 9e4 > 65504
        b = ones(m_in, np.float16)
        mid = np.full(k, 4096.0, np.float16)
        a = np.full(n, 2.0 ** -12, np.float16)
    else:
        raise ValueError(case)
    return Layer(dbf, A, B, a, mid, b, x)


EDGE_CASES = ["x_b_overflows_fp16", "x_b_subnormal_fp16", "mid_t_overflows_fp16"]


@pytest.mark.parametrize("case", EDGE_CASES)
def test_fused_decode_handles_the_ends_of_the_fp16_range(dbf, case):
    L = _edge_layer(dbf, case)
    ref = L.oracle()
    assert np.all(np.isfinite(ref)) and np.abs(ref).max() < 65504
    y = L.forward(flags=PATHS["decode_fused"], y_dtype=torch.float32).cpu().numpy()
    assert_fp16_close(y, ref, f"fused {case}")


@pytest.mark.parametrize("case", EDGE_CASES)
def test_prefill_path_at_the_ends_of_the_fp16_range(dbf, case):
    """b is folded into the sign tile exactly (x (.) b never rounds); V is fp16."""
    L = _edge_layer(dbf, case, batch=40)
    ref = L.oracle()
    y = L.forward(flags=PATHS["prefill"], y_dtype=torch.float32).cpu().numpy()
    if case == "mid_t_overflows_fp16":
        assert not np.all(np.isfinite(y)), "V = fp16(mid t) overflows to inf on this path"
    else:
        assert_fp16_close(y, ref, f"prefill {case}")


@pytest.mark.parametrize("case", EDGE_CASES)
def test_two_stage_decode_rounds_x_b_and_v_to_fp16(dbf, case):
    """The two-launch decode forms fp16(x (.) b) and fp16(mid t): overflow gives
    non-finite outputs, fp16 subnormals lose the relative precision the bar asks for."""
    L = _edge_layer(dbf, case)
    ref = L.oracle()
    y = L.forward(flags=PATHS["decode_class"], y_dtype=torch.float32).cpu().numpy()
    if case == "x_b_subnormal_fp16":
        rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
        assert np.all(np.isfinite(y)) and rel > 2e-3
    else:
        assert not np.all(np.isfinite(y))


def test_lost_arrival_reports_timeout_and_workspace_recovers(dbf):
    """A bounded wait that runs out: the kernel ends, the status word says so,
    and a zeroed workspace gives a correct forward on the same stream."""
    L = random_layer(dbf, 512, 512, 1024, 2, seed=21, scales="lognormal")
    ws = dbf.dbf_new_workspace(L.n, L.k, L.m_in, 2)
    y = torch.full((2, L.n), float("nan"), dtype=torch.float16, device="cuda")
    dbf.dbf_forward(L.x, L.pA, L.pB, L.a, L.mid, L.b, L.n, L.k, L.m_in, y=y, workspace=ws,
                    flags=PATHS["decode_fused"] | TEST_LOSE_ARRIVAL)
    torch.cuda.synchronize()
    assert dbf.dbf_workspace_status(ws) == DBF_ERR_TIMEOUT
    ws.zero_()
    y = L.forward(flags=PATHS["decode_fused"], workspace=ws)
    assert dbf.dbf_workspace_status(ws) == 0
    assert_fp16_close(y.float().cpu().numpy(), L.oracle(), "after a timeout")


def test_fused_decode_is_deterministic(dbf):
    L = random_layer(dbf, 1000, 1024, 2048, 5, seed=8, scales="lognormal")
    ys = [L.forward(flags=PATHS["decode_fused"], y_dtype=torch.float32) for _ in range(3)]
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])


@pytest.mark.parametrize("batch", [1, 2, 3, 6, 11, 16, 33])
def test_fused_decode_batches_integer_exact(dbf, batch):
    """Every N-tile count of the kernel (3 digit columns per token, 8 columns per
    tile) and chunks of 16 tokens past 16, bit-exact on integer data."""
    n, k, m_in = 300, 768, 1536
    rng = np.random.default_rng(batch)
    A, B = gen.sign_matrix(rng, n, k), gen.sign_matrix(rng, k, m_in)
    x = gen.integer_activations(rng, batch, m_in, -1, 1)
    ones = np.ones
    L = Layer(dbf, A, B, ones(n, np.float16), ones(k, np.float16), ones(m_in, np.float16), x)
    y = L.forward(flags=PATHS["decode_fused"], y_dtype=torch.float32).cpu().numpy().astype(np.float64)
    assert np.array_equal(y, L.oracle())


def test_fused_decode_exact_beyond_fp16_middle_range(dbf):
    """Integer data whose middle vector exceeds 2048 (fp16 would round it): the
    fused path keeps it exact, so y equals the integer result."""
    n, k, m_in = 128, 256, 4096
    rng = np.random.default_rng(3)
    A, B = gen.sign_matrix(rng, n, k), gen.sign_matrix(rng, k, m_in)
    B[:, :] = 1
    x = np.ones((1, m_in), np.float16)
    x[0, 0] = 0  # t = 4095 for every middle row: not an fp16 value (fp16 rounds it to 4096)
    ones = np.ones
    L = Layer(dbf, A, B, ones(n, np.float16), ones(k, np.float16), ones(m_in, np.float16), x)
    y = L.forward(flags=PATHS["decode_fused"], y_dtype=torch.float32).cpu().numpy().astype(np.float64)
    assert np.array_equal(y, L.oracle())
