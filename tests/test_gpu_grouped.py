"""GPU parity of dbf_forward_grouped: layers that share their input x, each
checked against the fp64 oracle's forward of that layer ("Addition is almost
all you need", gist.science technical summary, section 2.1), with the bars of
test_gpu_parity.py: bit-exact in integer mode, relative Frobenius error
<= 2e-3 and max error <= 1e-2 * rms on fp16 data."""
import numpy as np
import pytest
import torch

import dbf_inputs as gen
import oracle
from test_gpu_parity import PATHS, assert_fp16_close, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dbf():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from binary_factorized_weight_b200 import build

    build.build()
    import binary_factorized_weight_b200 as mod

    mod.load_library()
    return mod


def make_group(dbf, shapes, m_in, batch, seed, integer=False):
    """shapes: [(n, k), ...] sharing m_in; returns (x numpy, layers for the binding, numpy factors)."""
    rng = np.random.default_rng(seed)
    if integer:
        # |t| <= 2048 keeps the fp16 middle vector exact
        lim = max(1, min(8, 2048 // m_in))
        x = rng.integers(-lim, lim + 1, size=(batch, m_in)).astype(np.float16)
    else:
        x = gen.normal_activations(rng, batch, m_in)
    layers, facts = [], []
    for n, k in shapes:
        A = gen.sign_matrix(rng, n, k)
        B = gen.sign_matrix(rng, k, m_in)
        if integer:
            a, mid, b = gen.unit_scales(n), gen.unit_scales(k), gen.unit_scales(m_in)
        else:
            a, mid, b = gen.lognormal_scales(rng, n), gen.lognormal_scales(rng, k), gen.lognormal_scales(rng, m_in)
        facts.append(dict(A=A, B=B, a=a, mid=mid, b=b))
        layers.append(dict(packedA=dbf.dbf_pack_signs(dev(A)), packedB=dbf.dbf_pack_signs(dev(B)), a=dev(a),
                           m=dev(mid), b=dev(b), n=n, k=k))
    return x, layers, facts


SMALL = [(256, 128), (64, 64), (128, 192)]


@pytest.mark.parametrize("path", ["default", "decode_class", "decode_shift", "decode_table", "prefill"])
@pytest.mark.parametrize("batch", [1, 5, 16, 20, 200])
def test_grouped_integer_bit_exact(dbf, path, batch):
    x, layers, facts = make_group(dbf, SMALL, 256, batch, seed=7, integer=True)
    flags = 0 if path == "default" else PATHS[path]
    ys = dbf.dbf_forward_grouped(dev(x), layers, 256, y_dtype=torch.float32, flags=flags)
    torch.cuda.synchronize()
    for g, f in enumerate(facts):
        ref = oracle.forward_staged(x, f["A"], f["B"], f["a"], f["mid"], f["b"])
        assert np.array_equal(ys[g].cpu().numpy().astype(np.float64), ref), f"layer {g}"


@pytest.mark.parametrize("path", ["default", "decode_class", "decode_table", "prefill"])
@pytest.mark.parametrize("batch", [1, 9, 16, 130])
def test_grouped_fp16(dbf, path, batch):
    x, layers, facts = make_group(dbf, SMALL, 256, batch, seed=11)
    flags = 0 if path == "default" else PATHS[path]
    ys = dbf.dbf_forward_grouped(dev(x), layers, 256, flags=flags)
    torch.cuda.synchronize()
    for g, f in enumerate(facts):
        ref = oracle.forward_staged(x, f["A"], f["B"], f["a"], f["mid"], f["b"])
        assert_fp16_close(ys[g].float().cpu().numpy(), ref, f"layer {g}")


def test_grouped_matches_single_layer_calls_integer(dbf):
    """Grouping changes the launch, not the result: integer mode is identical to dbf_forward per layer."""
    x, layers, facts = make_group(dbf, [(128, 64), (64, 128), (192, 64)], 128, 3, seed=5, integer=True)
    xd = dev(x)
    ys = dbf.dbf_forward_grouped(xd, layers, 128, y_dtype=torch.float32)
    for g, L in enumerate(layers):
        y1 = dbf.dbf_forward(xd, L["packedA"], L["packedB"], L["a"], L["m"], L["b"], L["n"], L["k"], 128,
                             y_dtype=torch.float32)
        torch.cuda.synchronize()
        assert torch.equal(ys[g], y1), f"layer {g}"


def test_grouped_single_layer_equals_forward(dbf):
    x, layers, facts = make_group(dbf, [(256, 128)], 256, 4, seed=3)
    xd = dev(x)
    (yg,) = dbf.dbf_forward_grouped(xd, layers, 256)
    L = layers[0]
    # the grouped decode runs the two-launch kernels: the same arithmetic as dbf_forward's two-launch path
    y1 = dbf.dbf_forward(xd, L["packedA"], L["packedB"], L["a"], L["m"], L["b"], L["n"], L["k"], 256,
                         flags=dbf.DBF_FWD_DECODE_TWO_STAGE)
    torch.cuda.synchronize()
    assert torch.equal(yg, y1)


# Llama-style projections that share their input (1 and 2 bits/weight)
FULL = {
    "qkv_1b": [(4096, 2048), (1024, 832), (1024, 832)],
    "qkv_2b": [(4096, 4096), (1024, 1664), (1024, 1664)],
    "gate_up_1b": [(14336, 3200), (14336, 3200)],
}


@pytest.mark.parametrize("name", sorted(FULL))
@pytest.mark.parametrize("batch", [1, 16])
def test_grouped_full_size(dbf, name, batch):
    x, layers, facts = make_group(dbf, FULL[name], 4096, batch, seed=21)
    ys = dbf.dbf_forward_grouped(dev(x), layers, 4096, flags=dbf.DBF_FWD_WEIGHTS_STATIC)
    torch.cuda.synchronize()
    rows = np.arange(batch) if batch <= 4 else np.array([0, batch // 2, batch - 1])
    for g, f in enumerate(facts):
        ref = oracle.forward_staged(x[rows], f["A"], f["B"], f["a"], f["mid"], f["b"])
        assert_fp16_close(ys[g].float().cpu().numpy()[rows], ref, f"{name} layer {g}")


def test_grouped_workspace_status_stays_zero(dbf):
    x, layers, facts = make_group(dbf, SMALL, 256, 16, seed=2)
    ws = dbf.dbf_new_grouped_workspace(layers, 256, 16)
    dbf.dbf_forward_grouped(dev(x), layers, 256, workspace=ws)
    assert dbf.dbf_workspace_status(ws) == 0
