"""GPU parity of the one-token decode by table lookup (DBF_FWD_DECODE_TABLE).

The forward ("Addition is almost all you need", gist.science technical
summary section 2.1) is computed with one table per nibble of packed signs:
the 16 signed sums of the four activations those sign bits select, so a row's
product is one table entry per nibble.  The tables are fp32 sums of
u = x (.) b formed in fp32; the middle vector is still rounded to fp16 once.
  * integer mode (a = m = b = 1, integer x, fp32 output): bit-exact on ragged
    shapes (rows not a multiple of 64, K not a multiple of 256, several
    register groups and several pieces of K per CTA);
  * fp16 data: the usual bar against the oracle, on the workloads' layer
    shapes and on K long enough for several pieces;
  * fp16 range: x (.) b beyond 65504 or below the fp16 normal range is exact
    here (u is never rounded to fp16), while a middle vector beyond 65504 still
    overflows (V is fp16);
  * agreement with the default warp-MMA form within the bar, and determinism.
"""
import numpy as np
import pytest
import torch

from test_gpu_fused import _edge_layer
from test_gpu_parity import PATHS, assert_fp16_close, dbf, random_layer  # noqa: F401  (fixture)

pytestmark = pytest.mark.gpu

TABLE = PATHS["decode_table"]
MMA = PATHS["decode_class"]


@pytest.mark.parametrize("y_dtype", [torch.float32, torch.float16])
@pytest.mark.parametrize("n,k,m_in", [(100, 64, 64), (1000, 832, 4096), (333, 1664, 2880), (4096, 2048, 4096),
                                      (257, 448, 65536)])
def test_integer_bit_exact(dbf, n, k, m_in, y_dtype):
    x_lo = -1 if m_in > 8192 else -8  # |t| must stay <= 2048 for the fp16 middle vector
    L = random_layer(dbf, n, k, m_in, 1, seed=n + k, scales="unit", x_kind="int")
    if m_in > 8192:
        rng = np.random.default_rng(7)
        L.np["x"] = rng.integers(x_lo, -x_lo + 1, size=(1, m_in)).astype(np.float16)
        L.x = torch.from_numpy(L.np["x"]).cuda()
    ref = L.oracle()
    if y_dtype == torch.float16:
        ref = ref.astype(np.float16).astype(np.float64)  # the exact integer, rounded once to fp16
    y = L.forward(flags=TABLE, y_dtype=y_dtype).float().cpu().numpy().astype(np.float64)
    assert np.array_equal(y, ref)


@pytest.mark.parametrize("n,k,m_in", [(4096, 2048, 4096), (14336, 4736, 4096), (1024, 832, 4096),
                                      (4096, 3200, 14336), (512, 1024, 65536)])
def test_fp16_against_oracle(dbf, n, k, m_in):
    L = random_layer(dbf, n, k, m_in, 1, seed=3 * n + k, scales="lognormal")
    y = L.forward(flags=TABLE).float().cpu().numpy()
    assert_fp16_close(y, L.oracle(), f"table decode {n}x{k}x{m_in}")
    y2 = L.forward(flags=TABLE).float().cpu().numpy()
    assert np.array_equal(y, y2)  # deterministic


def test_table_against_warp_mma(dbf):
    """The default forward at one token is the warp-MMA form; the table kernel
    differs from it (the MMA form rounds x (.) b to fp16) and is no less
    accurate against the oracle."""
    L = random_layer(dbf, 1024, 1024, 2048, 1, seed=4, scales="lognormal")
    y_def = L.forward(flags=0, y_dtype=torch.float32).cpu().numpy()
    y_tab = L.forward(flags=TABLE, y_dtype=torch.float32).cpu().numpy()
    y_mma = L.forward(flags=MMA, y_dtype=torch.float32).cpu().numpy()
    assert np.array_equal(y_def, y_mma)
    assert not np.array_equal(y_tab, y_mma)
    ref = L.oracle()
    assert_fp16_close(y_mma, ref, "warp-MMA form")
    err_tab = np.linalg.norm(y_tab - ref) / np.linalg.norm(ref)
    err_mma = np.linalg.norm(y_mma - ref) / np.linalg.norm(ref)
    assert err_tab <= err_mma * 1.05  # no fp16 rounding of x (.) b: no less accurate


@pytest.mark.parametrize("case", ["x_b_overflows_fp16", "x_b_subnormal_fp16"])
def test_fp16_range_of_x_b_is_exact_here(dbf, case):
    L = _edge_layer(dbf, case, batch=1)
    y = L.forward(flags=TABLE, y_dtype=torch.float32).cpu().numpy()
    assert np.all(np.isfinite(y))
    assert_fp16_close(y, L.oracle(), case)


def test_middle_vector_overflow_still_shows(dbf):
    L = _edge_layer(dbf, "mid_t_overflows_fp16", batch=1)
    y = L.forward(flags=TABLE, y_dtype=torch.float32).cpu().numpy()
    assert not np.all(np.isfinite(y))


def test_graph_replay_and_status(dbf):
    L = random_layer(dbf, 4096, 2048, 4096, 1, seed=9, scales="unit", x_kind="int")
    ws = dbf.dbf_new_workspace(L.n, L.k, L.m_in, 1)
    y = torch.empty((1, L.n), dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    L.dbf.dbf_forward(L.x, L.pA, L.pB, L.a, L.mid, L.b, L.n, L.k, L.m_in, y=y, workspace=ws, flags=1 | TABLE,
                      stream=s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for _ in range(3):
            L.dbf.dbf_forward(L.x, L.pA, L.pB, L.a, L.mid, L.b, L.n, L.k, L.m_in, y=y, workspace=ws,
                              flags=1 | TABLE, stream=s)
    ref = L.oracle()
    for _ in range(2):
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(y.cpu().numpy().astype(np.float64), ref)
    assert dbf.dbf_workspace_status(ws) == 0
    del g
