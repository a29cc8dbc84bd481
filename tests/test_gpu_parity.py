"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Bars (the forward of "Addition is almost all you need", gist.science
technical summary section 2.1):
  * integer mode (a = m = b = 1, integer x, fp32 output, |t| <= 2048):
    bit-exact on every path;
  * fp16 data: relative Frobenius error <= 2e-3 and max |error| <= 1e-2 * rms(y);
  * packing: bit-exact words against the oracle's encoder, and the oracle's
    decoder recovers the signs.
Every output of every token is checked, at the full sizes too (the OpenMP
oracle takes well under a minute for the largest, 2048 tokens of the layer set).
"""
import numpy as np
import pytest
import torch

import dbf_inputs as gen
import oracle

pytestmark = pytest.mark.gpu

REL_FRO = 2e-3
MAX_REL_RMS = 1e-2


@pytest.fixture(scope="module")
def dbf():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from binary_factorized_weight_b200 import build

    build.build()
    import binary_factorized_weight_b200 as mod

    mod.load_library()
    return mod


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def assert_fp16_close(y, ref, what=""):
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    err = y - ref
    rel = np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300)
    rms = np.sqrt(np.mean(ref * ref))
    mx = np.abs(err).max()
    assert rel <= REL_FRO, f"{what}: relative Frobenius error {rel:.3e} > {REL_FRO}"
    assert mx <= MAX_REL_RMS * rms, f"{what}: max error {mx:.3e} > 1e-2 * rms {rms:.3e}"


class Layer:
    """A layer on the device: packed signs, scales, inputs."""

    def __init__(self, dbf, A, B, a, mid, b, x):
        self.dbf = dbf
        self.np = dict(A=A, B=B, a=a, mid=mid, b=b, x=x)
        self.n, self.k = A.shape
        self.m_in = B.shape[1]
        self.pA = dbf.dbf_pack_signs(dev(A))
        self.pB = dbf.dbf_pack_signs(dev(B))
        self.a, self.mid, self.b = dev(a), dev(mid), dev(b)
        self.x = dev(x)

    def forward(self, flags=0, y_dtype=torch.float16, x=None, workspace=None):
        x = self.x if x is None else x
        y = self.dbf.dbf_forward(x, self.pA, self.pB, self.a, self.mid, self.b, self.n, self.k, self.m_in,
                                 y_dtype=y_dtype, flags=flags, workspace=workspace)
        torch.cuda.synchronize()
        return y

    def oracle(self, rows=None):
        x = self.np["x"] if rows is None else self.np["x"][rows]
        return oracle.forward_staged(x, self.np["A"], self.np["B"], self.np["a"], self.np["mid"], self.np["b"])


def random_layer(dbf, n, k, m_in, batch, seed, scales="absnormal", x_kind="normal"):
    rng = np.random.default_rng(seed)
    A = gen.sign_matrix(rng, n, k)
    B = gen.sign_matrix(rng, k, m_in)
    if scales == "unit":
        a, mid, b = gen.unit_scales(n), gen.unit_scales(k), gen.unit_scales(m_in)
    elif scales == "lognormal":
        a, mid, b = gen.lognormal_scales(rng, n), gen.lognormal_scales(rng, k), gen.lognormal_scales(rng, m_in)
    else:
        a, mid, b = gen.abs_normal_scales(rng, n), gen.abs_normal_scales(rng, k), gen.abs_normal_scales(rng, m_in)
    x = gen.integer_activations(rng, batch, m_in) if x_kind == "int" else gen.normal_activations(rng, batch, m_in)
    return Layer(dbf, A, B, a, mid, b, x)


PATHS = {
    "decode_fused": 2 | 32,  # + DBF_FWD_DECODE_SINGLE: the single-launch int8 kernel where the shape fits
    "decode_class": 2 | 16,  # + DBF_FWD_DECODE_TWO_STAGE: two launches, fp16 class form
    "decode_table": 2 | 16 | 64,  # + DBF_FWD_DECODE_TABLE: two launches, one token by table lookup (class form above)
    "decode_shift": 2 | 8,  # + DBF_FWD_DECODE_SHIFT_EXPAND (two launches, shift form)
    "prefill": 4,  # DBF_FWD_FORCE_PREFILL
}


# ------------------------------------------------------------------ packing
@pytest.mark.parametrize("rows,cols", [(1, 1), (3, 64), (17, 128), (5, 200), (64, 832), (33, 4096)])
@pytest.mark.parametrize("dtype", [torch.int8, torch.float16, torch.float32])
def test_pack_bit_exact(dbf, rows, cols, dtype):
    rng = np.random.default_rng(rows * 1000 + cols)
    s = gen.sign_matrix(rng, rows, cols)
    src = dev(s).to(dtype)
    packed = dbf.dbf_pack_signs(src)
    torch.cuda.synchronize()
    words = packed.cpu().numpy().view(np.uint32)
    assert np.array_equal(words, oracle.pack_signs(s))
    back, bad = oracle.unpack_signs(words, rows, cols)
    assert bad == 0 and np.array_equal(back, s)


def test_pack_special_values(dbf):
    vals = torch.tensor([[0.0, -0.0, float("nan"), -float("nan"), float("inf"), -float("inf"), -1e-30, 1e-30] * 8],
                        dtype=torch.float32).cuda()
    expect = np.array([[1, 1, 1, 1, 1, -1, -1, 1] * 8], dtype=np.int8)
    for dt in (torch.float32, torch.float16):
        packed = dbf.dbf_pack_signs(vals.to(dt).contiguous())
        torch.cuda.synchronize()
        back, bad = oracle.unpack_signs(packed.cpu().numpy().view(np.uint32), 1, 64)
        exp = expect.copy()
        if dt == torch.float16:
            exp[0, 6::8] = 1  # -1e-30 underflows to -0.0 in fp16, which packs to +1
        assert bad == 0 and np.array_equal(back, exp), dt


# ------------------------------------------------------------------ tiny configs
@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("batch", [1, 4, 9, 16, 17, 128, 300])
def test_tiny_fp16(dbf, path, batch):
    shape = gen.CONFIGS["tiny"]
    L = Layer(dbf, **gen.make_layer(shape, batch))
    y = L.forward(flags=PATHS[path])
    assert_fp16_close(y.float().cpu().numpy(), L.oracle(), f"tiny {path} b{batch}")


@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("batch", [1, 4, 16, 128, 2048])
def test_tiny_int_bit_exact(dbf, path, batch):
    shape = gen.CONFIGS["tiny_int"]
    L = Layer(dbf, **gen.make_layer(shape, batch))
    y = L.forward(flags=PATHS[path], y_dtype=torch.float32).cpu().numpy().astype(np.float64)
    ref = L.oracle()
    assert np.array_equal(y, ref), f"max diff {np.abs(y - ref).max()}"


def test_default_dispatch_matches_forced(dbf):
    shape = gen.CONFIGS["tiny_int"]
    for batch in (1, 16, 17, 256):
        L = Layer(dbf, **gen.make_layer(shape, batch))
        y = L.forward(y_dtype=torch.float32).cpu().numpy()
        assert np.array_equal(y, L.oracle()), batch


# ------------------------------------------------------------------ ragged shapes / edges
RAGGED = [
    (1, 64, 64, 1), (3, 64, 128, 2), (100, 192, 320, 3), (1000, 832, 1088, 5), (17, 320, 64, 8),
    (130, 128, 256, 9), (64, 1088, 192, 16), (257, 256, 512, 33), (129, 64, 64, 129), (300, 192, 832, 257),
]


@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("n,k,m_in,batch", RAGGED)
def test_ragged_int_bit_exact(dbf, path, n, k, m_in, batch):
    rng = np.random.default_rng(n * 7 + k * 3 + m_in + batch)
    A, B = gen.sign_matrix(rng, n, k), gen.sign_matrix(rng, k, m_in)
    # keep |t| <= 2048 so that the fp16 middle vector is exact: |x| <= 2048 / m_in
    lim = max(1, min(8, 2048 // m_in))
    x = gen.integer_activations(rng, batch, m_in, -lim, lim)
    ones = np.ones
    L = Layer(dbf, A, B, ones(n, np.float16), ones(k, np.float16), ones(m_in, np.float16), x)
    y = L.forward(flags=PATHS[path], y_dtype=torch.float32).cpu().numpy().astype(np.float64)
    assert np.array_equal(y, L.oracle())


@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("n,k,m_in,batch", RAGGED)
def test_ragged_fp16(dbf, path, n, k, m_in, batch):
    L = random_layer(dbf, n, k, m_in, batch, seed=n + k + m_in + batch, scales="lognormal")
    y = L.forward(flags=PATHS[path]).float().cpu().numpy()
    assert_fp16_close(y, L.oracle(), f"{path} {n}x{k}x{m_in} b{batch}")


# ------------------------------------------------------------------ activations staged in several pieces
# 16 tokens over K = 4096 do not fit the decode kernel's shared-memory budget
# at once when the K split leaves one CTA per row tile the whole row (k = 16384
# rows in the first product): the activations then come in pieces, each
# overwriting the b-scaled copy of the previous one.
@pytest.mark.parametrize("batch", [9, 16])
def test_decode_activation_pieces_int_bit_exact(dbf, batch):
    n, k, m_in = 64, 16384, 4096
    rng = np.random.default_rng(batch)
    A, B = gen.sign_matrix(rng, n, k), gen.sign_matrix(rng, k, m_in)
    x = gen.integer_activations(rng, batch, m_in, -1, 1)
    ones = np.ones
    L = Layer(dbf, A, B, ones(n, np.float16), ones(k, np.float16), ones(m_in, np.float16), x)
    _, v = oracle.forward_staged(x, A, B, L.np["a"], L.np["mid"], L.np["b"], return_v=True)
    assert np.abs(v).max() <= 2048, "the fp16 middle vector would not be exact"
    y = L.forward(flags=PATHS["decode_class"], y_dtype=torch.float32).cpu().numpy().astype(np.float64)
    assert np.array_equal(y, L.oracle())


def test_decode_activation_pieces_fp16(dbf):
    L = random_layer(dbf, 64, 16384, 4096, 16, seed=77, scales="lognormal")
    for path in ("decode_class", "decode_shift"):
        y = L.forward(flags=PATHS[path]).float().cpu().numpy()
        assert_fp16_close(y, L.oracle(), f"activation pieces {path}")


# ------------------------------------------------------------------ wave tail of the persistent GEMM
def _tail_rows(batch):
    """Output rows n for which the second product's persistent launch (128-row x
    256-token tiles, one tile per SM per wave) would end in a wave of n_tiles
    tiles: the last 128-row tile (ragged: 91 rows) then goes to a split-K launch
    of its own."""
    from math import gcd

    sms = torch.cuda.get_device_properties(0).multi_processor_count
    n_tiles = (batch + 255) // 256
    m_tiles = sms // gcd(n_tiles, sms) + 1
    return m_tiles * 128 - 37


@pytest.mark.parametrize("batch", [256, 2048])
def test_wave_tail_int_bit_exact(dbf, batch):
    n, k, m_in = _tail_rows(batch), 1024, 256  # K = 1024: the tail launch splits K 4 ways
    rng = np.random.default_rng(n + batch)
    A, B = gen.sign_matrix(rng, n, k), gen.sign_matrix(rng, k, m_in)
    x = gen.integer_activations(rng, batch, m_in, -8, 8)
    ones = np.ones
    L = Layer(dbf, A, B, ones(n, np.float16), ones(k, np.float16), ones(m_in, np.float16), x)
    y = L.forward(flags=PATHS["prefill"], y_dtype=torch.float32).cpu().numpy().astype(np.float64)
    assert np.array_equal(y, L.oracle())


@pytest.mark.parametrize("batch", [256, 2048])
def test_wave_tail_fp16(dbf, batch):
    n = _tail_rows(batch)
    L = random_layer(dbf, n, 1024, 256, batch, seed=n + batch + 1, scales="lognormal")
    y = L.forward(flags=PATHS["prefill"]).float().cpu().numpy()
    assert_fp16_close(y, L.oracle(), f"wave tail {n}x1024x256 b{batch}")


def test_fp32_output_matches_fp16_output(dbf):
    L = random_layer(dbf, 256, 128, 256, 4, seed=3)
    for flags in PATHS.values():
        y16 = L.forward(flags=flags, y_dtype=torch.float16).cpu()
        y32 = L.forward(flags=flags, y_dtype=torch.float32).cpu()
        assert torch.equal(y32.half(), y16)


def test_negative_scales(dbf):
    rng = np.random.default_rng(11)
    n, k, m_in = 200, 256, 320
    A, B = gen.sign_matrix(rng, n, k), gen.sign_matrix(rng, k, m_in)
    a = (gen.abs_normal_scales(rng, n) * np.where(rng.random(n) < 0.5, -1, 1)).astype(np.float16)
    mid = (gen.abs_normal_scales(rng, k) * np.where(rng.random(k) < 0.5, -1, 1)).astype(np.float16)
    b = (gen.abs_normal_scales(rng, m_in) * np.where(rng.random(m_in) < 0.5, -1, 1)).astype(np.float16)
    for batch in (3, 150):
        L = Layer(dbf, A, B, a, mid, b, gen.normal_activations(rng, batch, m_in))
        for path, flags in PATHS.items():
            assert_fp16_close(L.forward(flags=flags).float().cpu().numpy(), L.oracle(), f"neg scales {path}")


# ------------------------------------------------------------------ closed forms / invariances
@pytest.mark.parametrize("p", [6, 8, 10])
def test_hadamard_closed_form_on_gpu(dbf, p):
    """A = B = Sylvester H_k, unit scales: H H = k I, so y = k x exactly."""
    size = 1 << p
    H = gen.sylvester_hadamard(p)
    rng = np.random.default_rng(p)
    ones = np.ones(size, np.float16)
    lim = max(1, 2048 // size)
    for batch in (1, 5, 200):
        x = gen.integer_activations(rng, batch, size, -lim, lim)
        L = Layer(dbf, H, H, ones, ones, ones, x)
        for path, flags in PATHS.items():
            y = L.forward(flags=flags, y_dtype=torch.float32).cpu().numpy()
            assert np.array_equal(y, size * x.astype(np.float32)), (path, batch)


def test_sign_flip_invariance_bit_exact(dbf):
    shape = gen.CONFIGS["tiny_int"]
    for batch in (4, 256):
        Ld = gen.make_layer(shape, batch)
        L1 = Layer(dbf, **Ld)
        A2, B2 = Ld["A"].copy(), Ld["B"].copy()
        cols = [0, 17, 64, 127]
        A2[:, cols] *= -1
        B2[cols, :] *= -1
        L2 = Layer(dbf, A2, B2, Ld["a"], Ld["mid"], Ld["b"], Ld["x"])
        for flags in PATHS.values():
            y1 = L1.forward(flags=flags, y_dtype=torch.float32)
            y2 = L2.forward(flags=flags, y_dtype=torch.float32)
            assert torch.equal(y1, y2)


# ------------------------------------------------------------------ reconstruction
@pytest.mark.parametrize("n,k,m_in", [(256, 128, 256), (100, 192, 320), (1000, 64, 64), (65, 832, 1088)])
def test_reconstruct_dense(dbf, n, k, m_in):
    L = random_layer(dbf, n, k, m_in, 1, seed=n * k, scales="lognormal")
    W = dbf.dbf_reconstruct_dense(L.pA, L.pB, L.a, L.mid, L.b, n, k, m_in, W_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = oracle.dense_weight(L.np["A"], L.np["B"], L.np["a"], L.np["mid"], L.np["b"])
    Wn = W.cpu().numpy().astype(np.float64)
    assert np.allclose(Wn, ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max())
    W16 = dbf.dbf_reconstruct_dense(L.pA, L.pB, L.a, L.mid, L.b, n, k, m_in, W_dtype=torch.float16)
    torch.cuda.synchronize()
    assert_fp16_close(W16.float().cpu().numpy(), ref, "reconstruct fp16")


def test_reconstruct_integer_exact(dbf):
    shape = gen.CONFIGS["tiny_int"]
    L = Layer(dbf, **gen.make_layer(shape, 1))
    W = dbf.dbf_reconstruct_dense(L.pA, L.pB, L.a, L.mid, L.b, L.n, L.k, L.m_in, W_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = oracle.dense_weight(L.np["A"], L.np["B"], L.np["a"], L.np["mid"], L.np["b"])
    assert np.array_equal(W.cpu().numpy().astype(np.float64), ref)


# ------------------------------------------------------------------ stream / PDL behaviour
@pytest.mark.parametrize("flags", [0, 1, 2, 3, 4, 5])
def test_chained_layers_read_fresh_inputs(dbf, flags):
    """Each forward reads the previous forward's output directly (PDL chain on one
    stream, no other kernel in between).  Constant scales 0.140625 keep the gain
    near 1 (0.14^3 * sqrt(512 * 256) ~ 1), so values stay O(1) over the chain."""
    n = m_in = 512
    k = 256
    batch = 200 if flags & 4 else 3
    rng = np.random.default_rng(42)
    A, B = gen.sign_matrix(rng, n, k), gen.sign_matrix(rng, k, m_in)
    c = np.float16(0.140625)
    L = Layer(dbf, A, B, np.full(n, c), np.full(k, c), np.full(m_in, c), gen.normal_activations(rng, batch, m_in))
    steps = 12
    ys = [L.x]
    ws = dbf.dbf_new_workspace(n, k, m_in, batch)
    for _ in range(steps):
        ys.append(dbf.dbf_forward(ys[-1], L.pA, L.pB, L.a, L.mid, L.b, n, k, m_in, workspace=ws, flags=flags))
    torch.cuda.synchronize()
    assert dbf.dbf_workspace_status(ws) == 0
    for i in range(steps):
        ref = oracle.forward_staged(ys[i].cpu().numpy(), A, B, L.np["a"], L.np["mid"], L.np["b"])
        assert np.sqrt(np.mean(ref * ref)) > 1e-3, "chain decayed; the check would be vacuous"
        assert_fp16_close(ys[i + 1].float().cpu().numpy(), ref, f"chain step {i}")


def test_cuda_graph_capture(dbf):
    L = random_layer(dbf, 384, 256, 512, 4, seed=9)
    ws = dbf.dbf_new_workspace(L.n, L.k, L.m_in, 4)
    y = torch.empty((4, L.n), dtype=torch.float16, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        dbf.dbf_forward(L.x, L.pA, L.pB, L.a, L.mid, L.b, L.n, L.k, L.m_in, y=y, workspace=ws, flags=1)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(3):
            dbf.dbf_forward(L.x, L.pA, L.pB, L.a, L.mid, L.b, L.n, L.k, L.m_in, y=y, workspace=ws, flags=1)
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert_fp16_close(y.float().cpu().numpy(), L.oracle(), "graph replay")


def test_workspace_status_stays_zero(dbf):
    L = random_layer(dbf, 256, 128, 256, 300, seed=1)
    ws = dbf.dbf_new_workspace(L.n, L.k, L.m_in, 300)
    for flags in PATHS.values():
        dbf.dbf_forward(L.x, L.pA, L.pB, L.a, L.mid, L.b, L.n, L.k, L.m_in, workspace=ws, flags=flags)
    assert dbf.dbf_workspace_status(ws) == 0


# ------------------------------------------------------------------ full-size workloads (every token)
FULL = [("attn_1b", 1), ("attn_2b", 1), ("attn_2b", 4), ("attn_2b", 16), ("mlp_up", 1), ("mlp_up", 2048)]


@pytest.mark.parametrize("name,batch", FULL)
def test_full_size_configs(dbf, name, batch):
    shape = gen.CONFIGS[name]
    L = Layer(dbf, **gen.make_layer(shape, batch))
    y = L.forward(flags=1).float().cpu().numpy()
    assert_fp16_close(y, L.oracle(), f"{name} b{batch}")  # every token


@pytest.mark.parametrize("bits", [1, 2])
@pytest.mark.parametrize("batch", [1, 16, 128, 2048])
def test_layer_set(dbf, bits, batch):
    for shape in gen.LAYER_SET[bits]:
        L = Layer(dbf, **gen.make_layer(shape, batch))
        y = L.forward(flags=1).float().cpu().numpy()
        assert_fp16_close(y, L.oracle(), f"{shape.name} b{batch}")  # every token
