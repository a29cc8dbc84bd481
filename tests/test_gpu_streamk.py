"""GPU parity of the stream-K schedule of the tensor-core path.

Past 128 tokens, when a GEMM's 256-token tiles do not fill whole waves of the
persistent grid and the workspace holds the stream-K area, the (tile,
256-column block) units are cut into one contiguous range per SM; a tile split
between CTAs is finished by the CTA holding its first blocks, which adds the
fp32 partial tiles of the others in CTA order.  The sums are the same products
as the plain schedule, only grouped differently, so:
  * integer mode (a = m = b = 1, integer x, fp32 output) is bit-exact against
    the oracle of the forward ("Addition is almost all you need", gist.science
    technical summary section 2.1) and identical to the plain schedule (run
    with a workspace too small for the stream-K area);
  * fp16 data meets the usual bar against the oracle;
  * the flags of the stream-K area are zero again after every call.
The planner takes stream-K where its estimated time beats the plain plan; the
shapes are chosen so that on a 148-SM B200 it does for one or both GEMMs, with
ragged rows, tokens and K, and tiles split over one to several CTAs.
"""
import numpy as np
import pytest
import torch

from test_gpu_parity import REL_FRO, assert_fp16_close, dbf, random_layer  # noqa: F401  (fixture)

pytestmark = pytest.mark.gpu

SK_FLAG_BYTES = 1024
SK_MAX_CTAS = 160
SK_SLOT_BYTES = 128 * 256 * 4


def v_area_end(k, batch):
    return 256 + (batch * k * 2 + 255) // 256 * 256


def cluster_split(M, K, batch, sms):
    """The K split of the plain plan for few 128-token tiles (1 = none)."""
    tiles128 = -(-M // 128) * -(-batch // 128)
    nblk = (K // 64 + 3) // 4
    if 2 * tiles128 > sms:
        return 1
    ks = 1
    while ks < 8 and tiles128 * ks * 2 <= sms and ks * 2 <= nblk:
        ks *= 2
    return ks


def takes_stream_k(M, K, batch, sms):
    """The planner's rule, restated: stream-K where units / SMs + 5 block times
    beats 0.95 of the plain plan's rounds x blocks per tile (a 128-token tile
    counted as 0.77 of a 256-token one, a cluster K slice as 1/ks)."""
    if batch <= 128:
        return False
    grid = min(sms, SK_MAX_CTAS)
    ks = cluster_split(M, K, batch, sms)
    m_tiles = -(-M // 128)
    ntile = 128
    if ks == 1:
        ntile = 128 if 2 * m_tiles * -(-batch // 256) <= sms else 256
    nblk = (K // 64 + 3) // 4
    units = m_tiles * -(-batch // 256) * nblk
    rounds = -(-(m_tiles * -(-batch // ntile) * ks) // sms)
    plan_t = rounds * nblk / ks * (0.77 if ntile == 128 else 1.0)
    return units >= grid and units / grid + 5.0 < 0.95 * plan_t


# (n, k, m_in, batch) and which GEMMs take stream-K on 148 SMs
SHAPES = [
    (2400, 2368, 2048, 2048),  # both GEMMs: 152 tiles each; ragged rows, a ragged last K block
    (9600, 2048, 2048, 300),   # the second GEMM: 150 tiles; a ragged 44-token last tile
    (1024, 832, 4096, 2048),   # k/v layer: the first GEMM, 56 tiles x 16 blocks, each tile over ~3 CTAs
]
EXPECT = {SHAPES[0]: (True, True), SHAPES[1]: (False, True), SHAPES[2]: (True, False)}


def sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


@pytest.mark.parametrize("n,k,m_in,batch", SHAPES)
def test_shapes_take_stream_k(dbf, n, k, m_in, batch):
    s = sms()
    if s != 148:
        pytest.skip("shape choice assumes 148 SMs")
    assert (takes_stream_k(k, m_in, batch, s), takes_stream_k(n, k, batch, s)) == EXPECT[(n, k, m_in, batch)]
    assert dbf.load_library().dbf_forward_workspace_bytes(n, k, m_in, batch) == \
        v_area_end(k, batch) + SK_FLAG_BYTES + SK_MAX_CTAS * SK_SLOT_BYTES


@pytest.mark.parametrize("y_dtype", [torch.float32, torch.float16])
@pytest.mark.parametrize("n,k,m_in,batch", SHAPES[:2])
def test_integer_bit_exact_and_same_as_plain_schedule(dbf, n, k, m_in, batch, y_dtype):
    L = random_layer(dbf, n, k, m_in, batch, seed=n + batch, scales="unit", x_kind="int")
    ws_full = torch.zeros(dbf.load_library().dbf_forward_workspace_bytes(n, k, m_in, batch), dtype=torch.uint8,
                          device="cuda")
    ws_min = torch.zeros(v_area_end(k, batch), dtype=torch.uint8, device="cuda")
    y_sk = L.forward(y_dtype=y_dtype, workspace=ws_full).float().cpu().numpy().astype(np.float64)
    y_plain = L.forward(y_dtype=y_dtype, workspace=ws_min).float().cpu().numpy().astype(np.float64)
    ref = L.oracle()
    if y_dtype == torch.float16:
        ref = ref.astype(np.float16).astype(np.float64)  # the exact integer, rounded once to fp16
    assert np.array_equal(y_sk, ref)
    assert np.array_equal(y_plain, ref)
    flags = ws_full[v_area_end(k, batch):v_area_end(k, batch) + SK_FLAG_BYTES]
    assert int(flags.count_nonzero()) == 0, "stream-K flags must be zero after the call"
    assert dbf.dbf_workspace_status(ws_full) == 0


@pytest.mark.parametrize("n,k,m_in,batch", SHAPES)
def test_fp16_against_oracle(dbf, n, k, m_in, batch):
    L = random_layer(dbf, n, k, m_in, batch, seed=3 * n + batch)
    ws = torch.zeros(dbf.load_library().dbf_forward_workspace_bytes(n, k, m_in, batch), dtype=torch.uint8,
                     device="cuda")
    y = L.forward(workspace=ws).float().cpu().numpy()
    if batch * (n * k + k * m_in) > 2048 * 8e6:
        rows = np.arange(0, batch, 5)  # every 5th token at the largest sizes (the oracle's time)
        assert_fp16_close(y[rows], L.oracle(rows), f"stream-K {n}x{k}x{m_in} b{batch}")
    else:
        assert_fp16_close(y, L.oracle(), f"stream-K {n}x{k}x{m_in} b{batch}")
    # repeated calls reuse the same zeroed flags
    y2 = L.forward(workspace=ws).float().cpu().numpy()
    assert np.array_equal(y, y2)
    assert dbf.dbf_workspace_status(ws) == 0


def test_fp16_close_to_plain_schedule(dbf):
    n, k, m_in, batch = SHAPES[0]
    L = random_layer(dbf, n, k, m_in, batch, seed=11)
    ws_full = torch.zeros(dbf.load_library().dbf_forward_workspace_bytes(n, k, m_in, batch), dtype=torch.uint8,
                          device="cuda")
    ws_min = torch.zeros(v_area_end(k, batch), dtype=torch.uint8, device="cuda")
    y_sk = L.forward(y_dtype=torch.float32, workspace=ws_full).cpu().numpy().astype(np.float64)
    y_plain = L.forward(y_dtype=torch.float32, workspace=ws_min).cpu().numpy().astype(np.float64)
    # only the grouping of the fp32 sums differs (V itself is rounded to fp16 from either)
    rel = np.linalg.norm(y_sk - y_plain) / np.linalg.norm(y_plain)
    assert rel < REL_FRO


def test_cuda_graph_replays_stream_k(dbf):
    n, k, m_in, batch = SHAPES[0]
    L = random_layer(dbf, n, k, m_in, batch, seed=12, scales="unit", x_kind="int")
    ws = torch.zeros(dbf.load_library().dbf_forward_workspace_bytes(n, k, m_in, batch), dtype=torch.uint8,
                     device="cuda")
    y = torch.empty((batch, n), dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    L.dbf.dbf_forward(L.x, L.pA, L.pB, L.a, L.mid, L.b, n, k, m_in, y=y, workspace=ws, stream=s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        L.dbf.dbf_forward(L.x, L.pA, L.pB, L.a, L.mid, L.b, n, k, m_in, y=y, workspace=ws, stream=s)
    ref = L.oracle()
    for _ in range(3):
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(y.cpu().numpy().astype(np.float64), ref)
    assert dbf.dbf_workspace_status(ws) == 0
    del g
